/*
 * bsa.h -- C ABI of the B200 (sm_100a) block-sparse attention library.
 *
 * Training-free, mean-pooled top-k block-sparse self-attention on a fixed
 * 128 (query rows) x 64 (key rows) block grid, in two stages:
 *
 *   (1) selection: mean-pool q over 128-row blocks and k over 64-row blocks,
 *       score the blocks with softmax(Qbar Kbar^T / sqrt(d)) per head, and keep
 *       the top-k fraction of key blocks for every query block;
 *   (2) attention: softmax attention that visits only the kept 128 x 64
 *       tiles (non-causal by default; is_causal != 0 restricts each row to
 *       keys at or before its own position).
 *
 * The calls mirror the interface on "SpargeAttention Documentation":
 * spas_sage2_attn_meansim_topk_cuda(q, k, v, topk, is_causal) (recommended API
 * paragraph) and block_sparse_sage2_attn_cuda(q, k, v, mask_id) with the mask
 * rules of its "Mask Requirements" section; the split into a selection call and
 * an apply call follows build_plan / apply_plan on the AB-Attention README
 * ("Use an existing pipeline", Q/K/V API).
 *
 * Conventions shared by every call
 *  - q, k, v, out: device pointers to contiguous bf16 tensors of shape
 *    [B, H, N, d] (row-major, d fastest), 16-byte aligned.  d is 64 or 128.
 *    out must not overlap q, k or v (BSA_ERR_INVALID_ARG).
 *  - Qb = ceil(N / 128), Kb = ceil(N / 64).  N <= 131072, so Kb <= 2048.
 *  - mask tensors are uint8 [B, H, Qb, Kb], row-major; nonzero means "keep".
 *  - ws: a device workspace of at least bsa_workspace_bytes(shape) bytes,
 *    256-byte aligned, owned by the caller.  The library never allocates device
 *    memory and keeps no per-call state between calls (sparse_attn_topk_host
 *    creates, and releases, five streams and their events per call); calls
 *    that share one workspace must be ordered on one stream.
 *  - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on it and returns after launching (for
 *    sparse_attn_topk_host the host buffers must stay valid until `stream` has
 *    been synchronised).  The device-buffer calls only enqueue work on `stream`
 *    and neither allocate nor synchronise, so they may be captured into a CUDA
 *    graph and replayed (sparse_attn_topk_host synchronises nothing either, but
 *    creates streams, so it is not meant for capture; bsa_last_device_status
 *    synchronises `stream`).
 *  - The attention scale is 1/sqrt(d), as in scaled-dot-product attention.
 *  - Errors: arguments are validated on the host before anything is launched;
 *    a rejected call returns BSA_ERR_INVALID_ARG or BSA_ERR_UNSUPPORTED and
 *    touches no memory.  A failed launch returns BSA_ERR_CUDA.  Every wait
 *    inside the attention and block-score kernels is bounded in time; if one
 *    runs out the kernel records it in ws and returns early, which
 *    bsa_last_device_status reports as BSA_ERR_TIMEOUT.  Every call that takes ws first clears that status word
 *    (on `stream`, before its kernels), so it always describes the latest call;
 *    a workspace that no call has used yet holds whatever its memory held.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1, /* bad shape, pointer, alignment, topk or workspace size */
  BSA_ERR_UNSUPPORTED = 2, /* an unsupported mode combination (is_causal with cdfthreshd) */
  BSA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  BSA_ERR_TIMEOUT = 4      /* a bounded wait inside a kernel ran out */
} bsa_status;

typedef struct {
  int32_t B; /* batch */
  int32_t H; /* heads */
  int32_t N; /* sequence length (tokens) */
  int32_t d; /* head dimension: 64 or 128 */
} bsa_shape;

/* Version of this ABI (incremented on incompatible changes). */
int bsa_abi_version(void);  /* 2: is_causal added to select / plan / apply */

/* Human-readable name of a status code (static string). */
const char* bsa_status_string(bsa_status s);

/* Detail of the last host-side rejection or CUDA error on the calling thread
 * (static, thread-local string; empty if none). */
const char* bsa_last_error_message(void);

/* Workspace bytes needed for a shape: pooled means, the fp32 block-score
 * matrix (B*H*Qb rows of Kb rounded up to 4 floats), the compacted per-query-
 * block key-block index list, its counts and the device status word.  Returns 0
 * for a shape the library rejects. */
size_t bsa_workspace_bytes(bsa_shape s);

/* Compressed block-score map.  Writes p_out, fp32 [B, H, Qb, Kb] (device),
 * with p_out[b,h,i,:] = softmax_j(Qbar_i . Kbar_j / sqrt(d)), where Qbar_i is
 * the mean of q rows [128 i, min(128 i + 128, N)) and Kbar_j the mean of k rows
 * [64 j, min(64 j + 64, N)) (means over valid rows only).  This is the score
 * that the top-k selection ranks. */
bsa_status sparse_attn_block_scores(const void* q, const void* k, bsa_shape s, float* p_out,
                                    void* ws, size_t ws_bytes, void* stream);

/* Selection stage.  Writes mask_out (device, uint8 [B, H, Qb, Kb]) with exactly
 * kk = clamp(ceil(topk * Kb), 1, Kb) ones per (b, h, i) row: the kk key blocks
 * with the largest block score, equal scores going to the lower block index.
 * kk is evaluated in double precision on the float value of topk.
 * topk must lie in (0, 1].  With is_causal != 0, row i chooses only among its
 * E_i = min(2 i + 2, Kb) causally eligible key blocks (blocks that hold a key
 * at or before some row of query block i) and keeps clamp(ceil(topk * E_i), 1,
 * E_i) of them; the other entries of the row are 0. */
bsa_status sparse_attn_select(const void* q, const void* k, bsa_shape s, float topk, int is_causal,
                              uint8_t* mask_out, void* ws, size_t ws_bytes, void* stream);

/* cdfthreshd selection (the "--mode cdfthreshd" option next to "topk" on
 * "SpargeAttention Documentation"; the pages print no formula, so this is a
 * reading): per (b, h, i) row, order the key blocks by block score descending
 * (equal scores: lower index first) and keep the shortest prefix whose
 * softmax mass reaches `threshold` (its float value, in (0, 1]); at least one
 * block; every block if rounding leaves the row's total mass below threshold.
 * Writes mask_out (device, uint8 [B, H, Qb, Kb]) and the plan in ws. */
bsa_status sparse_attn_select_cdf(const void* q, const void* k, bsa_shape s, float threshold,
                                  uint8_t* mask_out, void* ws, size_t ws_bytes, void* stream);

/* cdfthreshd selection followed by attention (the fused counterpart of
 * sparse_attn_topk for the cdfthreshd mode).  mask_out is optional.  This mode
 * is non-causal only: is_causal != 0 returns BSA_ERR_UNSUPPORTED. */
bsa_status sparse_attn_cdf(const void* q, const void* k, const void* v, bsa_shape s, float threshold,
                           int is_causal, void* out, uint8_t* mask_out, void* ws,
                           size_t ws_bytes, void* stream);

/* Attention over caller-chosen tiles.  mask_id (device, uint8 [B, H, Qb, Kb];
 * NULL means all ones, i.e. dense attention) selects the kept 128 x 64 tiles.
 * For every query row r of block i: out[r] = sum over kept tiles j and key rows
 * c < N of block j of softmax_c(q_r . k_c / sqrt(d)) v_c, the softmax taken
 * over the union of the kept keys.  A query block that keeps no key block gets
 * an all-zero output.  Rows >= N are never written.  With is_causal != 0 only
 * keys c <= r take part (mask entries past block 2 i + 1 are ignored and the
 * two diagonal blocks are masked element by element); a row left without any
 * key gets a zero output. */
bsa_status block_sparse_attn_fwd(const void* q, const void* k, const void* v, bsa_shape s,
                                 const uint8_t* mask_id, int is_causal, void* out,
                                 void* ws, size_t ws_bytes, void* stream);

/* Selection followed by attention in one call (three kernels on one stream,
 * no host synchronisation).  mask_out is optional (NULL: not written); when
 * given it receives the selection mask of sparse_attn_select.  is_causal has
 * the meaning of sparse_attn_select and block_sparse_attn_fwd. */
bsa_status sparse_attn_topk(const void* q, const void* k, const void* v, bsa_shape s, float topk,
                            int is_causal, void* out, uint8_t* mask_out, void* ws,
                            size_t ws_bytes, void* stream);

/* Plan / apply split (the build_plan / apply_plan pattern of the AB-Attention
 * README, "Use an existing pipeline"): the kept-block lists that
 * sparse_attn_select, sparse_attn_topk or block_sparse_attn_plan leave in ws
 * form a reusable plan.  block_sparse_attn_plan compacts a caller mask
 * (NULL = all ones) into ws without running attention. */
bsa_status block_sparse_attn_plan(const uint8_t* mask_id, bsa_shape s, int is_causal, void* ws,
                                  size_t ws_bytes, void* stream);

/* Attention over the plan currently held in ws (see block_sparse_attn_plan);
 * same output contract as block_sparse_attn_fwd.  The plan must have been
 * made for the same shape and the same is_causal; ws is not modified apart
 * from its status word. */
bsa_status block_sparse_attn_apply(const void* q, const void* k, const void* v, bsa_shape s,
                                   int is_causal, void* out, void* ws, size_t ws_bytes,
                                   void* stream);

/* No-allocation variant of sparse_attn_topk (same arguments minus the
 * workspace, is_causal included; same kernels, same results).  The pages have
 * no counterpart: this call exists for callers that cannot allocate device
 * memory, such as a serving engine that reserves all free device memory for its
 * own pool at start-up (so no memory is left for a workspace), or a caller on a
 * latency-critical path that must not trigger the device-wide synchronisation
 * of cudaFree.  Its scratch is a file-scope device array of 32 MiB, held on
 * every GPU that loads the library until the process exits.  The scratch holds
 * the block-score matrices of as many heads at a time as fit (the selection
 * then runs over the heads in chunks, with the same results); shapes whose
 * workspace with one head's score matrix exceeds 32 MiB are rejected with
 * BSA_ERR_INVALID_ARG before anything is launched.  The first call on a device
 * looks up that device's copy of the array with cudaGetSymbolAddress (with the
 * device current) and caches it per device and CUDA context (a new context,
 * after cudaDeviceReset for example, is looked up afresh), so make the first
 * call on each device, and the first after a reset, before any stream capture.
 * Every call on a device shares the one array, which keeps the last call's
 * contents: calls that may overlap on the GPU (different streams, other
 * threads) race and corrupt each other's results, so order them on one stream.
 * The call allocates nothing.  mask_out is optional (NULL: not written). */
bsa_status sparse_attn_topk_noalloc(const void* q, const void* k, const void* v, bsa_shape s,
                                    float topk, int is_causal, void* out, uint8_t* mask_out,
                                    void* stream);

/* Status of the last sparse_attn_topk_noalloc call on the current device, as
 * bsa_last_device_status reports it for a workspace: synchronises `stream`, then
 * returns BSA_OK, BSA_ERR_TIMEOUT (a bounded wait ran out and some output rows
 * were left unwritten) or BSA_ERR_CUDA.  No counterpart on the pages. */
bsa_status sparse_attn_topk_noalloc_status(void* stream);

/* sparse_attn_topk on HOST buffers, pipelined over chunks of heads: while the
 * attention of chunk c runs, chunk c+1's q/k/v are copied in on one internal
 * copy stream and chunk c-1's output is copied out on another.  Each chunk's
 * selection runs on a high-priority internal stream as soon as its inputs have
 * arrived, and the attention of consecutive chunks alternates between two
 * internal streams, so the next chunk's selection and first attention CTAs take
 * the SMs that the current chunk's last wave leaves idle.  The
 * pages have no counterpart: heads are independent (the same selection and
 * attention run per head), so this only overlaps PCIe transfers with the
 * compute of sparse_attn_topk, and out_host receives exactly the bytes that
 * sparse_attn_topk writes.
 *  - q_host, k_host, v_host (read), out_host (written): page-locked host memory
 *    (cudaHostAlloc / cudaHostRegister; anything else is BSA_ERR_INVALID_ARG),
 *    bf16 [B, H, N, d], 16-byte aligned.
 *  - q_dev, k_dev, v_dev, out_dev: device buffers of the same size, owned by the
 *    caller; the call overwrites all four.
 *  - ws, ws_bytes: a workspace for the full shape (bsa_workspace_bytes(s)).
 *    Each chunk's selection writes that chunk's heads of it, so afterwards it
 *    holds the kept-block lists of every head, as after sparse_attn_topk.
 *  - chunks: number of head chunks, clamped to [1, min(B*H, 64)], heads split
 *    evenly.  <= 0 picks about four waves of attention CTAs (one per SM) per
 *    chunk, with one head in the first and in the last chunk when there are at
 *    least two heads more than chunks (so the pipeline fills and drains with one
 *    head's copies).
 *  - stream: the compute stream.  Nothing starts before the work already queued
 *    on it, and it waits for the last copy out, so synchronising `stream` (then
 *    bsa_last_device_status) covers the whole call.  Non-causal and causal as in
 *    sparse_attn_topk; no mask is written.  The call creates five streams and
 *    their events and releases them when the work completes, so calls from
 *    several host threads do not share state. */
bsa_status sparse_attn_topk_host(const void* q_host, const void* k_host, const void* v_host,
                                 bsa_shape s, float topk, int is_causal, void* out_host, void* q_dev,
                                 void* k_dev, void* v_dev, void* out_dev, void* ws, size_t ws_bytes,
                                 int chunks, void* stream);

/* Token reordering (after the AB-Attention README's "Optional cube layout" and
 * the Morton3D ordering of the LightX2V page "Sol-Attn on Wan2.1"): writes
 * perm_out (host int32, text + T*Hg*Wg entries), perm[new] = old, for a
 * sequence of `text` tokens followed by a T x Hg x Wg video grid in raster
 * order.  Text tokens stay first and in place.  mode 0: raster (identity);
 * mode 1: 4 x 4 x 4 cubes, ordered by (t/4, h/4, w/4, t%4, h%4, w%4), cubes
 * clipped at the edges; mode 2: Morton3D, the key interleaving the bits of
 * (t, h, w).  Host only; no device memory is touched. */
bsa_status bsa_token_permutation(int T, int Hg, int Wg, int text, int mode, int32_t* perm_out);

/* Applies a token permutation to a contiguous [B, H, N, d] bf16 tensor:
 * dst[b, h, n] = src[b, h, perm[n]] (inverse = 0), or dst[b, h, perm[n]] =
 * src[b, h, n] (inverse != 0, undoing the first).  perm is a device int32
 * array of N entries that must be a permutation of 0..N-1 (not checked); src
 * and dst are distinct 16-byte aligned device buffers; d is a multiple of 8.
 * Asynchronous on `stream`. */
bsa_status bsa_permute_tokens(const void* src, void* dst, bsa_shape s, const int32_t* perm, int inverse,
                              void* stream);

/* Synchronises `stream`, then reports what the kernels of the last call that
 * used `ws` recorded: BSA_OK, BSA_ERR_TIMEOUT (a bounded wait ran out), or
 * BSA_ERR_CUDA if the stream holds an error.  A call whose wait ran out returns
 * BSA_OK itself (it only launches) and leaves some output rows unwritten, so a
 * caller that must know checks here after the call. */
bsa_status bsa_last_device_status(const void* ws, void* stream);

/* Limit of every bounded wait inside the kernels, in nanoseconds (process-wide;
 * default 1e10, i.e. 10 s; 0 restores the default; other values below 1000 are
 * raised to 1000).  The limit is measured on the GPU's global timer, which keeps
 * running while the context is time-sliced out by other work on a shared GPU,
 * so it is set far above any call's own duration (a CTA's longest wait is a few
 * microseconds in a healthy run); a lower limit risks reporting a timeout for a
 * call that was only preempted. */
void bsa_set_wait_timeout_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
