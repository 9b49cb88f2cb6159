// Block-sparse attention forward on sm_100a: only the kept 128 x 64 tiles of
// each (head, query block) are visited, following block_sparse_sage2_attn_cuda
// and its "Mask Requirements" ("SpargeAttention Documentation"): non-causal,
// bf16 inputs, scale 1/sqrt(d).
//
// Two kernels: bsa_fwd_kernel below (d = 128, and d = 64 when built with
// BSA_D64_TWO_CTA=0) and bsa_fwd1_kernel (d = 64, two CTAs per SM, one softmax
// warpgroup each; measured 5-9% faster at d = 64).
//
// bsa_fwd_kernel: one CTA per (head, query block), 384 threads in three warpgroups:
//   WG0  warp 0: TMA producer for the Q tile and the kept K tiles
//        warp 1: TMEM owner; one thread issues the Q K^T tcgen05.mma
//        warp 2: TMA producer for the kept V tiles
//        warp 3: one thread issues the P V tcgen05.mma
//        (the two issuers touch disjoint TMEM -- S buffers vs O accumulators
//        -- and synchronise only through the softmax barriers)
//   WG1, WG2: softmax.  Kept key blocks are consumed in pairs (128 keys); WG1
//        takes the even pairs and WG2 the odd ones.  Thread t of a softmax
//        warpgroup owns query row t, which is TMEM lane t, so row max / row
//        sum need no shuffles.
// Per pair j, S = Q K^T is one M=128, N=128 tcgen05 tile (N=64 for an odd last
// block) in the S buffer of warpgroup w = j % 2.  The warpgroup copies S into
// registers and releases the buffer at once, so the tensor core computes
// S_{j+2} while the exponentials of pair j run.  P (bf16) goes to a per-
// warpgroup tile -- in TMEM for d = 64, where P.V then reads its A operand
// from TMEM; in shared memory (K-major, 128-byte swizzle) for d = 128, whose
// O accumulators leave no TMEM room -- and O_w += P V accumulates in TMEM.  Each warpgroup keeps its own running max,
// row sum and O accumulator; the two are merged in the epilogue.
// The online softmax works in the exp2 domain and only rescales O when the row
// maximum grows by more than 2^8, which keeps every exponent <= 2^8 and is
// exact because l and O always share the same reference maximum.  A quarter of
// the exponentials run on the FMA pipes (exp2_poly2), the rest on MUFU.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "bsa_internal.h"

namespace bsa {
namespace {

// Column pairs c with bit (c % 8) set use the FMA-pipe exp2 polynomial; the
// others use MUFU ex2.  Measured on B200 against 0, 1/8, 1/4, 3/8 and 1/2:
// d = 128 is fastest with one pair in four (0x88), d = 64 in the two-warpgroup
// kernel with three in eight (0xA8).  The one-warpgroup d = 64 kernel, whose two
// CTAs on an SM exponentiate independently, is fastest with one or two pairs in
// eight (0x80, 0x82, 0x88 within 0.5% of each other, 0xA8 2.5% slower, 0 1%).
#ifndef BSA_POLY_PATTERN
#define BSA_POLY_PATTERN 0x88
#endif
#ifndef BSA_POLY_PATTERN_D64
#define BSA_POLY_PATTERN_D64 0xA8
#endif
#ifndef BSA_POLY_PATTERN_1WG
#define BSA_POLY_PATTERN_1WG 0x88
#endif

enum WaitSite : uint32_t {
  kWaitQ = 1,
  kWaitKFull = 2,
  kWaitKEmpty = 3,
  kWaitVFull = 4,
  kWaitVEmpty = 5,
  kWaitSFull = 6,
  kWaitPFull = 7,
  kWaitODone = 8,
  kWaitSFree = 9,
  kWaitPFree = 10,
};

struct AttnArgs {
  const int16_t* idx;  // [BH, Qb, Kb] kept key blocks, ascending, first cnt valid
  const int32_t* cnt;  // [BH, Qb]
  __nv_bfloat16* out;  // [BH, N, D]
  DeviceStatus* status;
  uint64_t timeout_ns;
  int N, Qb, Kb;
  int causal;        // keys after a row's own position are masked out (kernel template flag)
  float scale_log2;  // log2(e) / sqrt(d)
};

template <int D>
struct Cfg {
  static constexpr int kThreads = 384;
  static constexpr int kChunk = 16384;           // one 128-row x 64-column bf16 SW128 chunk
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 128 * D * 2;   // a pair of 64-row key blocks
  // With d = 64 the P tiles fit in TMEM next to S and O, and P.V reads its A
  // operand from there; with d = 128 TMEM is full and P goes through shared
  // memory.
  static constexpr bool kPTmem = D == 64;
  static constexpr int kKSt = (D == 128) ? 2 : 4;
  static constexpr int kVSt = (D == 128) ? 2 : 4;
  static constexpr int kPBytes = 128 * 128 * 2;  // one warpgroup's P tile (shared memory)
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKSt * kKVBytes;
  static constexpr int kOffP = kOffV + kVSt * kKVBytes;  // P tiles, or the epilogue exchange
  static constexpr int kSmem = kOffP + (kPTmem ? 2048 : 2 * kPBytes) + 1024;  // + alignment slack
  // TMEM columns: S buffer w at 128 w, O_w at 256 + D w, P_w at 384 + 64 w.
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColP = 384;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr unsigned kPolyPattern = (D == 64) ? BSA_POLY_PATTERN_D64 : BSA_POLY_PATTERN;
  // Registers per thread: the control warpgroup needs few; the softmax rows
  // hold 128 scores plus 64 packed P words.  40 / 232 measured ~1% faster than
  // 56 / 224; without setmaxnreg (168 for all) the kernel is ~30% slower.
  static constexpr uint32_t kRegCtl = 40;
  static constexpr uint32_t kRegSm = 232;
  static_assert(kSmem + 512 <= 227 * 1024, "shared memory budget (dynamic + static)");
  static_assert(kSmem > 114 * 1024, "one CTA per SM (it allocates all 512 TMEM columns)");
  static_assert(128 * kRegCtl + 256 * kRegSm <= 168 * 384, "register split must fit the launch budget");
};

// kCausal selects the diagonal masking at compile time, so the non-causal
// kernel carries none of its code (it measured ~5% slower with a runtime flag).
template <int D, bool kCausal>
__global__ void __launch_bounds__(384, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[C::kKSt], bar_kempty[C::kKSt],
      bar_vfull[C::kVSt], bar_vempty[C::kVSt], bar_sfull[2], bar_sfree[2], bar_pfull[2],
      bar_pfree[2], bar_odone, bar_qkdone;
  __shared__ uint32_t s_tmem;
  __shared__ int s_cnt, s_fail;
  __shared__ int s_tail[4];  // the last four kept key blocks (diagonal blocks are among them)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.Qb;
  const int qi = blockIdx.x - bh * a.Qb;
  const size_t row_id = static_cast<size_t>(bh) * a.Qb + qi;
  const int rows_valid = min(kBlockQ, a.N - qi * kBlockQ);
  const int16_t* idx_row = a.idx + row_id * a.Kb;
  __nv_bfloat16* out_blk = a.out + (static_cast<size_t>(bh) * a.N + static_cast<size_t>(qi) * kBlockQ) * D;

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const uint32_t sQ = base;
  const uint32_t sK0 = base + C::kOffK;
  const uint32_t sV0 = base + C::kOffV;
  const uint32_t sP0 = base + C::kOffP;

  // Thread 0 initialises the barriers and reads the count (and whether an
  // earlier CTA already gave up) while warp 1 allocates TMEM; every thread then
  // takes the same early-exit decision.
  if (threadIdx.x == 0) {
    const int c = (*reinterpret_cast<volatile uint32_t*>(&a.status->code) != 0) ? -1 : a.cnt[row_id];
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < C::kKSt; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int s = 0; s < C::kVSt; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(smem_u32(&bar_sfull[w]), 1);
      mbar_init(smem_u32(&bar_sfree[w]), 128);
      mbar_init(smem_u32(&bar_pfull[w]), 128);
      mbar_init(smem_u32(&bar_pfree[w]), 1);
    }
    mbar_init(smem_u32(&bar_odone), 1);
    mbar_init(smem_u32(&bar_qkdone), 1);
    fence_mbar_init();
    s_cnt = c;
    s_fail = 0;
    if (kCausal) {
#pragma unroll
      for (int t = 0; t < 4; ++t) s_tail[t] = (c - 4 + t >= 0) ? idx_row[c - 4 + t] : -1;
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int cnt = s_cnt;
  if (cnt <= 0) {
    if (cnt == 0) {  // no kept key block: the defined output is zero
      uint4* o4 = reinterpret_cast<uint4*>(out_blk);
      for (int e = threadIdx.x; e < rows_valid * D / 8; e += blockDim.x) o4[e] = make_uint4(0, 0, 0, 0);
    }
    if (warp == 1) tmem_dealloc(s_tmem, C::kTmemCols);
    return;
  }
  const uint32_t tmem = s_tmem;
  const int npairs = (cnt + 1) >> 1;
  DeviceStatus* st = a.status;
  const uint64_t tmo = a.timeout_ns;

  // Stage-issue counters, used by the producers to drain in-flight copies.
  static_assert(C::kKSt <= 4 && C::kVSt <= 4, "issued[] covers every ring stage");
  uint32_t issued[4] = {0, 0, 0, 0};
  bool mma_issued = false;

  if (warp < 4) {
    setmaxnreg_dec<C::kRegCtl>();
    if ((warp == 0 || warp == 2) && lane == 0) {
      // ---------------------------------------------- TMA producers
      // warp 0: Q, then the K tiles of every pair; warp 2: the V tiles.
      const bool is_k = warp == 0;
      const int nst = is_k ? C::kKSt : C::kVSt;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      const uint32_t ring = is_k ? sK0 : sV0;
      uint64_t* full = is_k ? bar_kfull : bar_vfull;
      uint64_t* empty = is_k ? bar_kempty : bar_vempty;
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(smem_u32(&bar_q), C::kQBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(sQ + c * C::kChunk, &tm_q, smem_u32(&bar_q), c * 64, qi * kBlockQ, bh);
        // The CTA that this SM is likely to run next (one per SM, dispatched in
        // order) starts with a Q tile from HBM; bring it into L2 now.
        uint32_t nsm;
        asm("mov.u32 %0, %%nsmid;" : "=r"(nsm));
        const unsigned nxt = blockIdx.x + nsm;
        if (nxt < gridDim.x) {
          const int nbh = static_cast<int>(nxt / a.Qb), nqi = static_cast<int>(nxt - nbh * a.Qb);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c) tma_prefetch_l2_3d(&tm_q, c * 64, nqi * kBlockQ, nbh);
        }
      }
      int b0 = __ldg(idx_row), b1 = cnt > 1 ? __ldg(idx_row + 1) : 0;
      for (int j = 0; j < npairs; ++j) {
        const int nx0 = 2 * j + 2 < cnt ? __ldg(idx_row + 2 * j + 2) : 0;  // next pair, prefetched
        const int nx1 = 2 * j + 3 < cnt ? __ldg(idx_row + 2 * j + 3) : 0;
        const int s = j % nst;
        const int n = j / nst;
        if (n > 0 && !mbar_wait(smem_u32(&empty[s]), (n - 1) & 1, st, tmo, is_k ? kWaitKEmpty : kWaitVEmpty)) break;
        const int nb = min(2, cnt - 2 * j);
        const uint32_t bar = smem_u32(&full[s]);
        mbar_expect_tx(bar, nb * 64 * D * 2);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(ring + s * C::kKVBytes + c * C::kChunk, map, bar, c * 64, b0 * kBlockK, bh);
        if (nb == 2) {
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(ring + s * C::kKVBytes + c * C::kChunk + 8192, map, bar, c * 64, b1 * kBlockK, bh);
        }
        ++issued[s];
        b0 = nx0;
        b1 = nx1;
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------- QK^T issuer
      // S_j = Q K_j^T into S buffer j % 2, once the softmax has copied S_{j-2}
      // out of that buffer.
      const uint64_t qd = sw128_desc(sQ, 16, 1024);
      bool ok = mbar_wait(smem_u32(&bar_q), 0, st, tmo, kWaitQ);
      mma_issued = true;
      for (int j = 0; ok && j < npairs; ++j) {
        const int w = j & 1;
        if (j >= 2 && !(ok = mbar_wait(smem_u32(&bar_sfree[w]), ((j - 2) >> 1) & 1, st, tmo, kWaitSFree))) break;
        const int s = j % C::kKSt;
        if (!(ok = mbar_wait(smem_u32(&bar_kfull[s]), (j / C::kKSt) & 1, st, tmo, kWaitKFull))) break;
        tc_fence_after();
        const int nb = min(2, cnt - 2 * j);
        const uint32_t idesc = idesc_bf16(128, 64 * nb, false);
        const uint32_t dt = tmem + C::kColS + w * 128;
        const uint64_t kd = sw128_desc(sK0 + s * C::kKVBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // descriptor start addresses advance in 16-byte units
          const uint32_t off = ((kk >> 2) * C::kChunk + (kk & 3) * 32) >> 4;
          umma_ss(dt, qd + off, kd + off, idesc, kk > 0);
        }
        umma_commit(smem_u32(&bar_sfull[w]));
        umma_commit(smem_u32(&bar_kempty[s]));
      }
      umma_commit(smem_u32(&bar_qkdone));
    } else if (warp == 3 && lane == 0) {
      // ---------------------------------------------- P.V issuer
      // O_w += P_j V_j (w = j % 2) once P_j is in shared memory.
      const uint32_t idesc_pv = idesc_bf16(128, D, true);
      bool ok = true;
      mma_issued = true;
      for (int j = 0; ok && j < npairs; ++j) {
        const int w = j & 1;
        if (!(ok = mbar_wait(smem_u32(&bar_pfull[w]), (j >> 1) & 1, st, tmo, kWaitPFull))) break;
        const int s = j % C::kVSt;
        if (!(ok = mbar_wait(smem_u32(&bar_vfull[s]), (j / C::kVSt) & 1, st, tmo, kWaitVFull))) break;
        tc_fence_after();
        const int nb = min(2, cnt - 2 * j);
        const uint64_t vd = sw128_desc(sV0 + s * C::kKVBytes, C::kChunk, 1024);
        const uint32_t od = tmem + C::kColO + w * D;
        const uint32_t acc0 = j >= 2 ? 1u : 0u;
        if constexpr (C::kPTmem) {
          // P_w: 128 lanes x 128 keys, two keys per column; 16 keys per step.
          const uint32_t pt = tmem + C::kColP + w * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            if (kk < nb * 4) umma_ts(od, pt + kk * 8, vd + kk * (2048 >> 4), idesc_pv, kk > 0 ? 1u : acc0);
          }
        } else {
          const uint64_t pd = sw128_desc(sP0 + w * C::kPBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            if (kk < nb * 4) {
              const uint32_t poff = ((kk >> 2) * C::kChunk + (kk & 3) * 32) >> 4;
              umma_ss(od, pd + poff, vd + kk * (2048 >> 4), idesc_pv, kk > 0 ? 1u : acc0);
            }
          }
        }
        umma_commit(smem_u32(&bar_pfree[w]));
        umma_commit(smem_u32(&bar_vempty[s]));
      }
      umma_commit(smem_u32(&bar_odone));
    }
  } else {
    setmaxnreg_inc<C::kRegSm>();
    // ------------------------------------------------ softmax warpgroups
    const int w = (warp >> 2) - 1;                   // 0: even pairs, 1: odd pairs
    const int row = threadIdx.x - 128 * (w + 1);     // query row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sbuf = tmem + lane_off + C::kColS + w * 128;
    const uint32_t obuf = tmem + lane_off + C::kColO + w * D;
    // Row `row` of this warpgroup's P tile (keys 0-63 in the first 16 KB
    // chunk, keys 64-127 in the second), K-major with the 128-byte swizzle.
    const uint32_t prow = sP0 + w * C::kPBytes + (row >> 3) * 1024 + (row & 7) * 128;
    const uint32_t pbuf = tmem + lane_off + C::kColP + w * 64;  // P_w in TMEM (d = 64)
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const int kb_last = a.Kb - 1;
    const int tail = a.N - kb_last * kBlockK;  // valid keys in the last key block (1..64)
    // The ragged last key block can only be the last kept one.
    const bool ragged = tail < 64 && __ldg(idx_row + cnt - 1) == kb_last;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int t = 0;
    for (int j = w; j < npairs; j += 2, ++t) {
      ok = mbar_wait(smem_u32(&bar_sfull[w]), t & 1, st, tmo, kWaitSFull);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const int nb = min(2, cnt - 2 * j);
      float s[128];
      tmem_ld128(sbuf, s);  // for an odd last block the upper 64 columns are stale and overwritten below
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_sfree[w]));  // S buffer may now receive S_{j+2}
      if (nb != 2) {
#pragma unroll
        for (int c = 64; c < 128; ++c) s[c] = -INFINITY;
      }
      if (ragged && j == npairs - 1) {  // the last kept block is the ragged last key block
        if (nb == 1) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = c >= tail ? -INFINITY : s[c];
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[64 + c] = c >= tail ? -INFINITY : s[64 + c];
        }
      }
      if (kCausal && 2 * j + 1 >= cnt - 4) {
        // Only the kept blocks 2 qi and 2 qi + 1 straddle the diagonal, and being
        // the highest kept indices they are among the last four.  Key column c of
        // block b is visible to row `row` when 64 b + c <= 128 qi + row.
        const int b0 = s_tail[2 * j - cnt + 4 < 0 ? 0 : 2 * j - cnt + 4];
        const int b1 = nb == 2 ? s_tail[2 * j + 1 - cnt + 4] : -1;
        const bool d0 = 2 * j - cnt + 4 >= 0 && b0 >= 2 * qi;
        const bool d1 = b1 >= 2 * qi;
        const int lim0 = row - (b0 - 2 * qi) * 64, lim1 = row - (b1 - 2 * qi) * 64;
        if (d0) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = c > lim0 ? -INFINITY : s[c];
        }
        if (d1) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[64 + c] = c > lim1 ? -INFINITY : s[64 + c];
        }
      }
      float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]);
      float mx2 = fmax3(s[6], s[7], s[8]), mx3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
      for (int c = 12; c < 124; c += 8) {
        mx0 = fmax3(mx0, s[c], s[c + 1]);
        mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
        mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
        mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
      }
      const float rmax = fmax3(fmax3(mx0, mx1, s[124]), fmax3(mx2, mx3, s[125]), fmaxf(s[126], s[127]));
      const float m_new = fmaxf(m_run, rmax * sl2);
      const bool need = m_new > m_run + 8.0f;  // always true for the first pair
      const float m_use = need ? m_new : m_run;
      // A row that has seen no visible key yet (possible only with causal
      // masking) keeps m = -inf, weight 0 and alpha 1.
      const bool dead = kCausal && m_use == -INFINITY;
      const float alpha = dead ? 1.f : ex2_approx(m_run - m_use);  // 0 for the first pair, 1 if no rescale
      const float m_ref = dead ? 0.f : m_use;
      const uint64_t negm = f2_pack(-m_ref, -m_ref);
      // Exponentials of column pairs: x = s * log2(e)/sqrt(d) - m as one f32x2
      // FMA; the pairs selected by C::kPolyPattern on the FMA-pipe polynomial,
      // the rest on MUFU.
      uint32_t pk[64];
      uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        if (c >= 32 && nb != 2) break;
        const uint64_t x = f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), sl2x2, negm);
        float x0, x1;
        f2_unpack(x, x0, x1);
        uint64_t pp;
        if ((C::kPolyPattern >> (c & 7)) & 1) {
          pp = exp2_poly2(x0, x1);
        } else {
          pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
        }
        acc[c & 1] = f2_add(acc[c & 1], pp);
        float p0, p1;
        f2_unpack(pp, p0, p1);
        pk[c] = pack_bf16(p0, p1);
      }
      float a0, a1, a2, a3;
      f2_unpack(acc[0], a0, a1);
      f2_unpack(acc[1], a2, a3);
      l_run = l_run * alpha + ((a0 + a1) + (a2 + a3));
      // P buffer and O_w are free once this warpgroup's previous P.V is done.
      if (t > 0) {
        ok = mbar_wait(smem_u32(&bar_pfree[w]), (t - 1) & 1, st, tmo, kWaitPFree);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            float o[32];
            tmem_ld32(obuf + cc * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(obuf + cc * 32, reinterpret_cast<const uint32_t*>(o));
          }
          tmem_wait_st();
        }
      }
      if constexpr (C::kPTmem) {
        tmem_st32(pbuf, pk);
        if (nb == 2) tmem_st32(pbuf + 32, pk + 32);
        tmem_wait_st();
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && nb != 2) break;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint32_t addr = prow + h * C::kChunk + ((g ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(pk[h * 32 + g * 4]), "r"(pk[h * 32 + g * 4 + 1]),
                         "r"(pk[h * 32 + g * 4 + 2]), "r"(pk[h * 32 + g * 4 + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();  // make P visible to the tensor core's async proxy
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull[w]));
      m_run = m_use;
    }
    // ---------------------------------------------- epilogue: merge O_0, O_1
    // Each warpgroup's (m, l) for its row go through shared memory (the P
    // tiles, idle once every P.V has completed); then warpgroup w writes
    // output columns [w D/2, (w+1) D/2) of its row.
    if (ok) {
      ok = mbar_wait(smem_u32(&bar_odone), 0, st, tmo, kWaitODone);
      ok = __all_sync(0xffffffffu, ok);
    }
    float* xch = reinterpret_cast<float*>(dsmem + (sP0 - smem_u32(dsmem)));  // [2][128] m, [2][128] l
    if (ok) {
      xch[w * 128 + row] = m_run;
      xch[256 + w * 128 + row] = l_run;
    } else if (lane == 0) {
      s_fail = 1;
    }
    named_bar_sync(1, 256);
    if (s_fail == 0) {
      tc_fence_after();
      const bool has1 = npairs > 1;  // warpgroup 1 saw at least one pair
      const float m0 = xch[row], m1 = xch[128 + row];
      const float m = has1 ? fmaxf(m0, m1) : m0;
      // m = -inf: the row saw no visible key (causal); its output is zero.
      const float a0 = (m == -INFINITY || m0 == -INFINITY) ? 0.f : ex2_approx(m0 - m);
      const float a1 = (!has1 || m == -INFINITY || m1 == -INFINITY) ? 0.f : ex2_approx(m1 - m);
      const float lsum = xch[256 + row] * a0 + (has1 ? xch[384 + row] * a1 : 0.f);
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      const float c0 = a0 * inv, c1 = a1 * inv;
      __nv_bfloat16* orow = out_blk + static_cast<size_t>(row) * D;
#pragma unroll 1
      for (int cc = w * (D / 64); cc < (w + 1) * (D / 64); ++cc) {
        float o0[32], o1[32];
        tmem_ld32(tmem + lane_off + C::kColO + cc * 32, o0);
        if (has1) {
          tmem_ld32(tmem + lane_off + C::kColO + D + cc * 32, o1);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o1[e] = 0.f;
        }
        uint32_t wv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          wv[e] = pack_bf16(fmaf(o0[2 * e], c0, o1[2 * e] * c1), fmaf(o0[2 * e + 1], c0, o1[2 * e + 1] * c1));
        if (row < rows_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  // Every role has left its loop (finished, or gave up after a bounded wait).
  // Drain what may still be in flight before the TMEM is released and the CTA
  // exits: outstanding TMA loads (producers) and tensor-core ops (issuers).
  // Those always finish within microseconds, so the drain waits up to at
  // least 100 ms even when the caller set a shorter wait limit.
  const uint64_t drain = tmo > 100000000ull ? tmo : 100000000ull;
  __syncthreads();
  if ((warp == 0 || warp == 2) && lane == 0) {
    const int nst = (warp == 0) ? C::kKSt : C::kVSt;
    for (int s = 0; s < nst; ++s) {
      if (issued[s] == 0) continue;
      const uint32_t bar = smem_u32(warp == 0 ? &bar_kfull[s] : &bar_vfull[s]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar, (issued[s] - 1) & 1)) {
        if (globaltimer_ns() - t0 > drain) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
    if (warp == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bar_q), 0)) {
        if (globaltimer_ns() - t0 > drain) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
  }
  if (warp == 1 || warp == 3) {
    if (lane == 0 && mma_issued) {
      // Each issuer committed a final barrier after its last MMA; wait for it (bounded).
      const uint32_t fin = smem_u32(warp == 1 ? &bar_qkdone : &bar_odone);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(fin, 0)) {
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
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------ d = 64: one softmax warpgroup per CTA
// At d = 64 the softmax chain, not the tensor core, bounds the kernel above.
// This variant runs TWO CTAs per SM, each with one query block, one softmax
// warpgroup and half of the TMEM (256 columns: S at 0, O at 128, P at 192), so
// the two softmax warpgroups of an SM are independent: each CTA has its own
// Q K^T and P V issuers (four per SM), no cross-warpgroup merge, and one CTA's
// prologue and epilogue overlap the other's pairs.  256 threads:
//   warps 0-3: softmax (thread t owns query row t, TMEM lane t);
//   warp 4: TMA producer for Q and the K tiles; warp 5: TMEM owner and Q K^T
//   issuer; warp 6: TMA producer for the V tiles; warp 7: P V issuer.
// Registers: launched at 128 per thread (two CTAs fill the register file);
// setmaxnreg gives the softmax 232 and the control warps 24.
struct Cfg1 {
  static constexpr int D = 64;
  static constexpr int kThreads = 256;
  static constexpr int kChunk = 16384;             // 128 rows x 64 bf16 columns, SW128
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 128 * D * 2;     // a pair of 64-row key blocks
  static constexpr int kKSt = 2;
  static constexpr int kVSt = 3;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKSt * kKVBytes;
  static constexpr int kSmem = kOffV + kVSt * kKVBytes + 1024;  // + alignment slack
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColO = 128;
  static constexpr uint32_t kColP = 192;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr unsigned kPolyPattern = BSA_POLY_PATTERN_1WG;
  static constexpr uint32_t kRegSm = 232;
  static constexpr uint32_t kRegCtl = 24;
  static_assert(2 * (kSmem + 1024 + 512) <= 228 * 1024, "two CTAs per SM (shared memory)");
  static_assert(128 * kRegSm + 128 * kRegCtl <= 128 * kThreads, "register split of the launch budget");
};

template <bool kCausal>
__global__ void __launch_bounds__(256, 2)
    bsa_fwd1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = Cfg1;
  constexpr int D = C::D;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bar_q, bar_kfull[C::kKSt], bar_kempty[C::kKSt], bar_vfull[C::kVSt],
      bar_vempty[C::kVSt], bar_sfull, bar_sfree, bar_pfull, bar_pfree, bar_odone, bar_qkdone;
  __shared__ uint32_t s_tmem;
  __shared__ int s_cnt;
  __shared__ int s_tail[4];  // the last four kept key blocks (diagonal blocks are among them)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x / a.Qb;
  const int qi = blockIdx.x - bh * a.Qb;
  const size_t row_id = static_cast<size_t>(bh) * a.Qb + qi;
  const int rows_valid = min(kBlockQ, a.N - qi * kBlockQ);
  const int16_t* idx_row = a.idx + row_id * a.Kb;
  __nv_bfloat16* out_blk = a.out + (static_cast<size_t>(bh) * a.N + static_cast<size_t>(qi) * kBlockQ) * D;

  const uint32_t base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const uint32_t sQ = base;
  const uint32_t sK0 = base + C::kOffK;
  const uint32_t sV0 = base + C::kOffV;

  if (threadIdx.x == 0) {
    const int c = (*reinterpret_cast<volatile uint32_t*>(&a.status->code) != 0) ? -1 : a.cnt[row_id];
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < C::kKSt; ++s) {
      mbar_init(smem_u32(&bar_kfull[s]), 1);
      mbar_init(smem_u32(&bar_kempty[s]), 1);
    }
    for (int s = 0; s < C::kVSt; ++s) {
      mbar_init(smem_u32(&bar_vfull[s]), 1);
      mbar_init(smem_u32(&bar_vempty[s]), 1);
    }
    mbar_init(smem_u32(&bar_sfull), 1);
    mbar_init(smem_u32(&bar_sfree), 128);
    mbar_init(smem_u32(&bar_pfull), 128);
    mbar_init(smem_u32(&bar_pfree), 1);
    mbar_init(smem_u32(&bar_odone), 1);
    mbar_init(smem_u32(&bar_qkdone), 1);
    fence_mbar_init();
    s_cnt = c;
    if (kCausal) {
#pragma unroll
      for (int t = 0; t < 4; ++t) s_tail[t] = (c - 4 + t >= 0) ? idx_row[c - 4 + t] : -1;
    }
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int cnt = s_cnt;
  if (cnt <= 0) {
    if (cnt == 0) {  // no kept key block: the defined output is zero
      uint4* o4 = reinterpret_cast<uint4*>(out_blk);
      for (int e = threadIdx.x; e < rows_valid * D / 8; e += blockDim.x) o4[e] = make_uint4(0, 0, 0, 0);
    }
    if (warp == 5) tmem_dealloc(s_tmem, C::kTmemCols);
    return;
  }
  const uint32_t tmem = s_tmem;
  const int npairs = (cnt + 1) >> 1;
  DeviceStatus* st = a.status;
  const uint64_t tmo = a.timeout_ns;
  // per ring stage, the loads issued into it (K and V share the counters)
  uint32_t issued[C::kKSt > C::kVSt ? C::kKSt : C::kVSt] = {};
  bool mma_issued = false;

  if (warp >= 4) {
    setmaxnreg_dec<C::kRegCtl>();
    if ((warp == 4 || warp == 6) && lane == 0) {
      // ---------------------------------------------- TMA producers
      const bool is_k = warp == 4;
      const int nst = is_k ? C::kKSt : C::kVSt;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      const uint32_t ring = is_k ? sK0 : sV0;
      uint64_t* full = is_k ? bar_kfull : bar_vfull;
      uint64_t* empty = is_k ? bar_kempty : bar_vempty;
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(smem_u32(&bar_q), C::kQBytes);
        tma_load_3d(sQ, &tm_q, smem_u32(&bar_q), 0, qi * kBlockQ, bh);
      }
      int b0 = __ldg(idx_row), b1 = cnt > 1 ? __ldg(idx_row + 1) : 0;
      for (int j = 0; j < npairs; ++j) {
        const int nx0 = 2 * j + 2 < cnt ? __ldg(idx_row + 2 * j + 2) : 0;
        const int nx1 = 2 * j + 3 < cnt ? __ldg(idx_row + 2 * j + 3) : 0;
        const int s = j % nst;
        const int n = j / nst;
        if (n > 0 && !mbar_wait(smem_u32(&empty[s]), (n - 1) & 1, st, tmo, is_k ? kWaitKEmpty : kWaitVEmpty)) break;
        const int nb = min(2, cnt - 2 * j);
        const uint32_t bar = smem_u32(&full[s]);
        mbar_expect_tx(bar, nb * 64 * D * 2);
        tma_load_3d(ring + s * C::kKVBytes, map, bar, 0, b0 * kBlockK, bh);
        if (nb == 2) tma_load_3d(ring + s * C::kKVBytes + 8192, map, bar, 0, b1 * kBlockK, bh);
        ++issued[s];
        b0 = nx0;
        b1 = nx1;
      }
    } else if (warp == 5 && lane == 0) {
      // ---------------------------------------------- QK^T issuer
      const uint64_t qd = sw128_desc(sQ, 16, 1024);
      bool ok = mbar_wait(smem_u32(&bar_q), 0, st, tmo, kWaitQ);
      mma_issued = true;
      for (int j = 0; ok && j < npairs; ++j) {
        if (j > 0 && !(ok = mbar_wait(smem_u32(&bar_sfree), (j - 1) & 1, st, tmo, kWaitSFree))) break;
        const int s = j % C::kKSt;
        if (!(ok = mbar_wait(smem_u32(&bar_kfull[s]), (j / C::kKSt) & 1, st, tmo, kWaitKFull))) break;
        tc_fence_after();
        const int nb = min(2, cnt - 2 * j);
        const uint32_t idesc = idesc_bf16(128, 64 * nb, false);
        const uint64_t kd = sw128_desc(sK0 + s * C::kKVBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) umma_ss(tmem + C::kColS, qd + kk * 2, kd + kk * 2, idesc, kk > 0);
        umma_commit(smem_u32(&bar_sfull));
        umma_commit(smem_u32(&bar_kempty[s]));
      }
      umma_commit(smem_u32(&bar_qkdone));
    } else if (warp == 7 && lane == 0) {
      // ---------------------------------------------- P.V issuer
      const uint32_t idesc_pv = idesc_bf16(128, D, true);
      bool ok = true;
      mma_issued = true;
      for (int j = 0; ok && j < npairs; ++j) {
        if (!(ok = mbar_wait(smem_u32(&bar_pfull), j & 1, st, tmo, kWaitPFull))) break;
        const int s = j % C::kVSt;
        if (!(ok = mbar_wait(smem_u32(&bar_vfull[s]), (j / C::kVSt) & 1, st, tmo, kWaitVFull))) break;
        tc_fence_after();
        const int nb = min(2, cnt - 2 * j);
        const uint64_t vd = sw128_desc(sV0 + s * C::kKVBytes, C::kChunk, 1024);
        const uint32_t acc0 = j >= 1 ? 1u : 0u;
        // P: 128 lanes x 128 keys, two keys per column; 16 keys per step.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          if (kk < nb * 4)
            umma_ts(tmem + C::kColO, tmem + C::kColP + kk * 8, vd + kk * (2048 >> 4), idesc_pv, kk > 0 ? 1u : acc0);
        umma_commit(smem_u32(&bar_pfree));
        umma_commit(smem_u32(&bar_vempty[s]));
      }
      umma_commit(smem_u32(&bar_odone));
    }
  } else {
    setmaxnreg_inc<C::kRegSm>();
    // ------------------------------------------------ softmax warpgroup
    const int row = threadIdx.x;  // query row in the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t sbuf = tmem + lane_off + C::kColS;
    const uint32_t obuf = tmem + lane_off + C::kColO;
    const uint32_t pbuf = tmem + lane_off + C::kColP;
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const int kb_last = a.Kb - 1;
    const int tail = a.N - kb_last * kBlockK;  // valid keys in the last key block (1..64)
    const bool ragged = tail < 64 && __ldg(idx_row + cnt - 1) == kb_last;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < npairs; ++j) {
      ok = mbar_wait(smem_u32(&bar_sfull), j & 1, st, tmo, kWaitSFull);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const int nb = min(2, cnt - 2 * j);
      float s[128];
      tmem_ld128_halves(sbuf, s);
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_sfree));  // the S buffer may now receive the next S
      if (nb != 2) {
#pragma unroll
        for (int c = 64; c < 128; ++c) s[c] = -INFINITY;
      }
      if (ragged && j == npairs - 1) {
        if (nb == 1) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = c >= tail ? -INFINITY : s[c];
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[64 + c] = c >= tail ? -INFINITY : s[64 + c];
        }
      }
      if (kCausal && 2 * j + 1 >= cnt - 4) {
        // Key column c of block b is visible to row `row` when 64 b + c <= 128 qi + row.
        const int b0 = s_tail[2 * j - cnt + 4 < 0 ? 0 : 2 * j - cnt + 4];
        const int b1 = nb == 2 ? s_tail[2 * j + 1 - cnt + 4] : -1;
        const bool d0 = 2 * j - cnt + 4 >= 0 && b0 >= 2 * qi;
        const bool d1 = b1 >= 2 * qi;
        const int lim0 = row - (b0 - 2 * qi) * 64, lim1 = row - (b1 - 2 * qi) * 64;
        if (d0) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = c > lim0 ? -INFINITY : s[c];
        }
        if (d1) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[64 + c] = c > lim1 ? -INFINITY : s[64 + c];
        }
      }
      float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]);
      float mx2 = fmax3(s[6], s[7], s[8]), mx3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
      for (int c = 12; c < 124; c += 8) {
        mx0 = fmax3(mx0, s[c], s[c + 1]);
        mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
        mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
        mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
      }
      const float rmax = fmax3(fmax3(mx0, mx1, s[124]), fmax3(mx2, mx3, s[125]), fmaxf(s[126], s[127]));
      const float m_new = fmaxf(m_run, rmax * sl2);
      const bool need = m_new > m_run + 8.0f;  // always true for the first pair
      const float m_use = need ? m_new : m_run;
      const bool dead = kCausal && m_use == -INFINITY;
      const float alpha = dead ? 1.f : ex2_approx(m_run - m_use);
      const float m_ref = dead ? 0.f : m_use;
      const uint64_t negm = f2_pack(-m_ref, -m_ref);
      uint32_t pk[64];
      uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        if (c >= 32 && nb != 2) break;
        const uint64_t x = f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), sl2x2, negm);
        float x0, x1;
        f2_unpack(x, x0, x1);
        uint64_t pp;
        if ((C::kPolyPattern >> (c & 7)) & 1) {
          pp = exp2_poly2(x0, x1);
        } else {
          pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
        }
        acc[c & 1] = f2_add(acc[c & 1], pp);
        float p0, p1;
        f2_unpack(pp, p0, p1);
        pk[c] = pack_bf16(p0, p1);
      }
      float a0, a1, a2, a3;
      f2_unpack(acc[0], a0, a1);
      f2_unpack(acc[1], a2, a3);
      l_run = l_run * alpha + ((a0 + a1) + (a2 + a3));
      // The P tile and O are free once the previous P.V is done.
      if (j > 0) {
        ok = mbar_wait(smem_u32(&bar_pfree), (j - 1) & 1, st, tmo, kWaitPFree);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            float o[32];
            tmem_ld32(obuf + cc * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(obuf + cc * 32, reinterpret_cast<const uint32_t*>(o));
          }
          tmem_wait_st();
        }
      }
      tmem_st32(pbuf, pk);
      if (nb == 2) tmem_st32(pbuf + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_pfull));
      m_run = m_use;
    }
    // ---------------------------------------------- epilogue: O / l
    if (ok) {
      ok = mbar_wait(smem_u32(&bar_odone), 0, st, tmo, kWaitODone);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      // m = -inf: the row saw no visible key (causal); its output is zero (its l
      // is not exactly 0: the polynomial exp2 returns ~1e-38 for -inf).
      const float inv = (m_run == -INFINITY || !(l_run > 0.f)) ? 0.f : 1.f / l_run;
      __nv_bfloat16* orow = out_blk + static_cast<size_t>(row) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(obuf + cc * 32, o);
        uint32_t wv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) wv[e] = pack_bf16(o[2 * e] * inv, o[2 * e + 1] * inv);
        if (row < rows_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  // As in bsa_fwd_kernel: drain the loads and MMAs that may still be in flight
  // (bounded, at least 100 ms), then release the TMEM.
  const uint64_t drain = tmo > 100000000ull ? tmo : 100000000ull;
  __syncthreads();
  if ((warp == 4 || warp == 6) && lane == 0) {
    const int nst = (warp == 4) ? C::kKSt : C::kVSt;
    for (int s = 0; s < nst; ++s) {
      if (issued[s] == 0) continue;
      const uint32_t bar = smem_u32(warp == 4 ? &bar_kfull[s] : &bar_vfull[s]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar, (issued[s] - 1) & 1)) {
        if (globaltimer_ns() - t0 > drain) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
    if (warp == 4) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bar_q), 0)) {
        if (globaltimer_ns() - t0 > drain) {
          atomicCAS(&st->code, 0u, kDevTimeout);
          break;
        }
      }
    }
  }
  if (warp == 5 || warp == 7) {
    if (lane == 0 && mma_issued) {
      const uint32_t fin = smem_u32(warp == 5 ? &bar_qkdone : &bar_odone);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(fin, 0)) {
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
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------- host side
// [BH, N, D] bf16 viewed as a 3-D tensor (D fastest); box = 64 columns x rows x 1,
// 128-byte swizzle, rows past N read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int BH, int N, int D, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
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

// The d = 64 kernel with one softmax warpgroup per CTA and two CTAs per SM
// (bsa_fwd1_kernel); 0 selects the two-warpgroup kernel for d = 64 as well.
#ifndef BSA_D64_TWO_CTA
#define BSA_D64_TWO_CTA 1
#endif

template <bool kCausal>
cudaError_t launch_one_wg(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const AttnArgs& args, int BH, cudaStream_t st) {
  auto kern = bsa_fwd1_kernel<kCausal>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg1::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(BH) * static_cast<unsigned>(args.Qb);
  kern<<<grid, Cfg1::kThreads, Cfg1::kSmem, st>>>(mq, mk, mv, args);
  return cudaGetLastError();
}

template <int D, bool kCausal>
cudaError_t launch_typed(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const AttnArgs& args, int BH, cudaStream_t st) {
  if (D == 64 && BSA_D64_TWO_CTA) return launch_one_wg<kCausal>(mq, mk, mv, args, BH, st);
  using C = Cfg<D>;
  auto kern = bsa_fwd_kernel<D, kCausal>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(BH) * static_cast<unsigned>(args.Qb);
  kern<<<grid, C::kThreads, C::kSmem, st>>>(mq, mk, mv, args);
  return cudaGetLastError();
}

}  // namespace

EncodeTiledFn encode_tiled_fn() {
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

cudaError_t launch_attention(const void* q, const void* k, const void* v, void* out, int BH, int N,
                             int d, int causal, const int16_t* idx, const int32_t* cnt,
                             DeviceStatus* status, uint64_t timeout_ns, cudaStream_t st,
                             const char** why) {
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
  args.causal = causal ? 1 : 0;
  args.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(d));
  if (d == 128)
    return causal ? launch_typed<128, true>(mq, mk, mv, args, BH, st)
                  : launch_typed<128, false>(mq, mk, mv, args, BH, st);
  return causal ? launch_typed<64, true>(mq, mk, mv, args, BH, st)
                : launch_typed<64, false>(mq, mk, mv, args, BH, st);
}

}  // namespace bsa
