// Block dot products S[bh][i][j] = Qbar_i . Kbar_j on the tensor cores.
//
// The selection ranks key blocks by these fp32 dot products, and its masks must
// match an fp64 reference except where two block scores lie within 1e-6 of
// each other, so the product needs fp32-like accuracy.  TF32 alone keeps 11
// significant bits; here every operand x is split into hi = x rounded to TF32
// and lo = x - hi (rounded to TF32 as well), and each product is accumulated as
// hi*hi + hi*lo + lo*hi (the lo*lo term is below 2^-22 of the product).  In
// fp32 the three products of a K = 8 step land in one fp32 accumulator in TMEM.
// Measured against fp64 on the video-shaped workloads this is as accurate as
// fp32 FMA accumulation (relative error ~1e-6 of |Qbar_i| |Kbar_j|, no ranking
// change outside the 1e-6 band).
//
// Persistent: one CTA per SM walks the tiles of 128 query blocks x 256 key
// blocks (all heads), 384 threads:
//   warp 0: TMA producer (32-wide fp32 chunks of Qbar and Kbar, 128-byte swizzle);
//   warp 1: TMEM owner and MMA issuer (tcgen05.mma kind::tf32, M 128, N 256, K 8);
//   warps 4-7: split each chunk into hi and lo in shared memory (elementwise, so
//              the swizzled layout is kept);
//   warps 8-11: epilogue, TMEM -> shared staging (32 columns at a time, 128-byte
//               swizzle) -> bulk tensor stores into S (rows past Qb and
//               columns past Kp clipped by the store).
// The operand ring has two stages of 96 KB (A hi, A lo, B hi, B lo) and runs on
// across tiles; two TMEM accumulators of 256 columns let a tile's epilogue
// overlap the next tile's loads, splits and MMAs.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa_internal.h"

namespace bsa {
namespace {

constexpr int kTcM = 128;      // query blocks per tile (MMA M, TMEM lanes)
constexpr int kTcN = 256;      // key blocks per tile (MMA N, TMEM columns)
constexpr int kTcKc = 32;      // fp32 elements of d per chunk (one 128-byte swizzle row)
constexpr int kTcThreads = 384;
constexpr int kTcStages = 2;
constexpr int kTcABytes = kTcM * kTcKc * 4;                   // 16 KB
constexpr int kTcBBytes = kTcN * kTcKc * 4;                   // 32 KB
constexpr int kTcStageBytes = 2 * (kTcABytes + kTcBBytes);    // A hi | A lo | B hi | B lo
constexpr int kTcOutBytes = kTcM * 32 * 4;                   // one 32-column slab of a tile: 16 KB
constexpr int kTcSmem = kTcStages * kTcStageBytes + 2 * kTcOutBytes + 1024;  // + alignment slack
static_assert(kTcSmem + 128 <= 227 * 1024, "shared memory budget (dynamic + static)");
constexpr uint32_t kTcTmemCols = 512;            // two accumulators

// Wait sites recorded in the device status word (the attention kernel uses 1-10).
enum : uint32_t { kWaitTcFull = 21, kWaitTcConv = 22, kWaitTcEmpty = 23, kWaitTcAccFull = 24, kWaitTcAccEmpty = 25 };

// tcgen05.mma kind::tf32 instruction descriptor: fp32 D, TF32 A and B, both
// K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4)                                  // D format: f32
         | (2u << 7)                                // A format: tf32
         | (2u << 10)                               // B format: tf32
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Bulk tensor store shared -> global of one box at (x, y, z); completion is
// tracked per thread with bulk groups.
__device__ __forceinline__ void tma_store_3d(const void* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Waits until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// x -> (hi, lo): hi = x rounded to the 10 explicit mantissa bits of TF32 (ties
// away from zero in magnitude), lo = x - hi (exact in fp32) rounded the same
// way.  The tensor core reads only the TF32 bits of each 32-bit operand.
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  hi = __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
  lo = __uint_as_float((__float_as_uint(x - hi) + 0x1000u) & 0xFFFFE000u);
}

// Splits n float4 of `raw` in place (hi) and into `lo`, thread t of the
// converter warpgroup taking elements t, t + 128, ...
__device__ __forceinline__ void split_tile(float4* raw, float4* lo, int n, int t) {
  for (int e = t; e < n; e += 128) {
    const float4 x = raw[e];
    float4 h, l;
    split_tf32(x.x, h.x, l.x);
    split_tf32(x.y, h.y, l.y);
    split_tf32(x.z, h.z, l.z);
    split_tf32(x.w, h.w, l.w);
    raw[e] = h;
    lo[e] = l;
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    dots_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_s, int nI, int nJ, int ntiles, DeviceStatus* st,
                   uint64_t tmo) {
  constexpr int kChunks = D / kTcKc;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_full[kTcStages], bar_conv[kTcStages], bar_empty[kTcStages],
      bar_accfull[2], bar_accempty[2], bar_done;
  __shared__ uint32_t s_tmem;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  uint8_t* const gbase = dsmem + (base - smem_u32(dsmem));  // generic pointer to `base`
  // tile t: key-block tile t % nJ, query-block tile (t / nJ) % nI, head t / (nJ nI)
  auto tile = [&](int t, int& i0, int& j0, int& bh) {
    j0 = (t % nJ) * kTcN;
    i0 = ((t / nJ) % nI) * kTcM;
    bh = t / (nJ * nI);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_conv[s]), 128);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(smem_u32(&bar_accfull[p]), 1);
      mbar_init(smem_u32(&bar_accempty[p]), 128);
    }
    mbar_init(smem_u32(&bar_done), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  uint32_t issued[kTcStages] = {};
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    int g = 0;  // chunk sequence number across tiles
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      int i0, j0, bh;
      tile(t, i0, j0, bh);
      for (int c = 0; c < kChunks; ++c, ++g) {
        const int s = g % kTcStages;
        const int n = g / kTcStages;
        if (n > 0 && !(ok = mbar_wait(smem_u32(&bar_empty[s]), (n - 1) & 1, st, tmo, kWaitTcEmpty))) break;
        const uint32_t sa = base + s * kTcStageBytes;
        const uint32_t bar = smem_u32(&bar_full[s]);
        mbar_expect_tx(bar, kTcABytes + kTcBBytes);
        tma_load_3d(sa, &tm_q, bar, c * kTcKc, i0, bh);                  // A: rows i0.. (past Qb: zeros)
        tma_load_3d(sa + 2 * kTcABytes, &tm_k, bar, c * kTcKc, j0, bh);  // B: rows j0.. (past Kb: zeros)
        ++issued[s];
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_tf32(kTcM, kTcN);
    mma_issued = true;
    bool ok = true;
    int g = 0, lt = 0;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++lt) {
      const int p = lt & 1;  // accumulator of this tile
      if (lt >= 2 && !(ok = mbar_wait(smem_u32(&bar_accempty[p]), ((lt >> 1) - 1) & 1, st, tmo, kWaitTcAccEmpty)))
        break;
      tc_fence_after();
      const uint32_t dt = tmem + p * kTcN;
      for (int c = 0; c < kChunks; ++c, ++g) {
        const int s = g % kTcStages;
        if (!(ok = mbar_wait(smem_u32(&bar_conv[s]), (g / kTcStages) & 1, st, tmo, kWaitTcConv))) break;
        tc_fence_after();
        const uint32_t sa = base + s * kTcStageBytes;
        const uint64_t ahi = sw128_desc(sa, 16, 1024);
        const uint64_t alo = sw128_desc(sa + kTcABytes, 16, 1024);
        const uint64_t bhi = sw128_desc(sa + 2 * kTcABytes, 16, 1024);
        const uint64_t blo = sw128_desc(sa + 2 * kTcABytes + kTcBBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kTcKc / 8; ++kk) {
          // K = 8 fp32 = 32 bytes per step; descriptor addresses count 16-byte units
          const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
          umma_tf32(dt, ahi + kk * 2, bhi + kk * 2, idesc, acc);
          umma_tf32(dt, ahi + kk * 2, blo + kk * 2, idesc, 1u);
          umma_tf32(dt, alo + kk * 2, bhi + kk * 2, idesc, 1u);
        }
        umma_commit(smem_u32(&bar_empty[s]));
      }
      if (!ok) break;
      umma_commit(smem_u32(&bar_accfull[p]));
    }
    umma_commit(smem_u32(&bar_done));
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ split
    const int tid = threadIdx.x - 128;
    int g = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
      for (int c = 0; c < kChunks; ++c, ++g) {
        const int s = g % kTcStages;
        ok = mbar_wait(smem_u32(&bar_full[s]), (g / kTcStages) & 1, st, tmo, kWaitTcFull);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        uint8_t* gs = gbase + s * kTcStageBytes;
        split_tile(reinterpret_cast<float4*>(gs), reinterpret_cast<float4*>(gs + kTcABytes), kTcABytes / 16, tid);
        split_tile(reinterpret_cast<float4*>(gs + 2 * kTcABytes),
                   reinterpret_cast<float4*>(gs + 2 * kTcABytes + kTcBBytes), kTcBBytes / 16, tid);
        fence_proxy_async_smem();  // the tensor core reads these tiles through the async proxy
        mbar_arrive(smem_u32(&bar_conv[s]));
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ epilogue
    // Thread (quarter q, lane l) holds TMEM lane 32 q + l = row 32 q + l of the
    // tile; per 32-column slab it writes its row into a staging buffer (16-byte
    // chunk c of row r at chunk c ^ (r % 8), the 128-byte swizzle the store map
    // expects, so each quarter-warp's stores hit eight different bank groups),
    // and one thread stores the slab.  Two staging buffers alternate.
    const int quarter = warp & 3;
    const int et = threadIdx.x - 256;  // 0..127
    const int r = 32 * quarter + lane;
    const uint32_t stage0 = base + kTcStages * kTcStageBytes;
    int lt = 0, slab = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int p = lt & 1;
      bool ok = mbar_wait(smem_u32(&bar_accfull[p]), (lt >> 1) & 1, st, tmo, kWaitTcAccFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      int i0, j0, bh;
      tile(t, i0, j0, bh);
      const uint32_t taddr = tmem + p * kTcN + (static_cast<uint32_t>(32 * quarter) << 16);
#pragma unroll 1
      for (int cc = 0; cc < kTcN / 32; ++cc, ++slab) {
        const uint32_t buf = stage0 + (slab & 1) * kTcOutBytes;
        if (slab >= 2) {
          if (et == 0) bulk_wait_read<1>();  // the store issued two slabs ago has read `buf`
          named_bar_sync(1, 128);
        }
        float v[32];
        tmem_ld32(taddr + cc * 32, v);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t a = buf + r * 128 + ((c ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v[4 * c]), "f"(v[4 * c + 1]),
                       "f"(v[4 * c + 2]), "f"(v[4 * c + 3])
                       : "memory");
        }
        fence_proxy_async_smem();  // the bulk store reads the buffer through the async proxy
        named_bar_sync(1, 128);
        if (et == 0) {
          tma_store_3d(&tm_s, buf, j0 + cc * 32, i0, bh);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_accempty[p]));  // accumulator p may take tile lt + 2
    }
    if (et == 0) bulk_wait_all();
  }

  // ---------------------------------------------------------------- teardown
  // Drain what may still be in flight (bounded, at least 100 ms) before the
  // TMEM is released: the producer's loads and the issuer's MMAs.
  const uint64_t drain = tmo > 100000000ull ? tmo : 100000000ull;
  __syncthreads();
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      if (issued[s] == 0) continue;
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bar_full[s]), (issued[s] - 1) & 1)) {
        if (globaltimer_ns() - t0 > drain) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
  }
  if (warp == 1) {
    if (lane == 0 && mma_issued) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bar_done), 0)) {
        if (globaltimer_ns() - t0 > drain) {
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
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

// [BH, rows, D] fp32 viewed as a 3-D tensor (D fastest); box = 32 columns x
// box_rows x 1, 128-byte swizzle; loads read rows past `rows` as zero, stores
// clip them (and columns past D).
bool make_map_f32(CUtensorMap* m, const float* ptr, int BH, int rows, int D, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4,
                                 static_cast<cuuint64_t>(rows) * D * 4};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kTcKc), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_dots_tc(const float* qbar, const float* kbar, int BH, int Qb, int Kb, int d,
                           float* S, DeviceStatus* status, uint64_t timeout_ns, cudaStream_t st) {
  CUtensorMap mq, mk, ms;
  const int Kp = padded_kb(Kb);
  if (!make_map_f32(&mq, qbar, BH, Qb, d, kTcM) || !make_map_f32(&mk, kbar, BH, Kb, d, kTcN) ||
      !make_map_f32(&ms, S, BH, Qb, Kp, kTcM))
    return cudaErrorInvalidValue;
  const int nJ = (Kb + kTcN - 1) / kTcN, nI = (Qb + kTcM - 1) / kTcM;
  const int64_t ntiles = static_cast<int64_t>(nJ) * nI * BH;
  if (ntiles > 0x7fffffff) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  const unsigned grid = static_cast<unsigned>(ntiles < sms ? ntiles : sms);  // one CTA per SM
  const int nt = static_cast<int>(ntiles);
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(dots_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
    if (e != cudaSuccess) return e;
    dots_tc_kernel<128><<<grid, kTcThreads, kTcSmem, st>>>(mq, mk, ms, nI, nJ, nt, status, timeout_ns);
  } else {
    e = cudaFuncSetAttribute(dots_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
    if (e != cudaSuccess) return e;
    dots_tc_kernel<64><<<grid, kTcThreads, kTcSmem, st>>>(mq, mk, ms, nI, nJ, nt, status, timeout_ns);
  }
  return cudaGetLastError();
}

}  // namespace bsa
