/*
 * sskip_attn.h -- C ABI of libsskip_attn.so: Skip-Softmax tiled attention on
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes
 * -------------------------
 * FlashAttention-style tiled attention in which a block of logits is skipped
 * when it sits far enough below the running maximum.  The TensorRT-LLM
 * Skip-Softmax article ("TRT-LLM sparse attention, 1.4x", section
 * "Skip Softmax 的三步走算法") gives the test in three steps: take the block's
 * local maximum logit; compare it with the running global maximum; when the
 * gap exceeds the threshold, skip the block's softmax, its second matmul
 * (P.V) and the load of its V block from HBM.  The same article ("实战演练"
 * section) defines the threshold as threshold_scale_factor divided by the
 * context length: t = threshold_scale_factor / L.
 *
 * Exactly:  for query-tile rows r and key tile j (visited in ascending j),
 *   m_local[r] = max over visible keys of sm_scale * q_r . k_c
 *   row r passes  iff  m_local[r] - m_run[r] < ln t     (strict; ln 0 = -inf)
 *   the tile is skipped iff every valid row passes; a skipped tile changes
 *   neither the running max m, nor the row sum l, nor the accumulator O;
 *   a kept tile runs the usual online-softmax update and O += P V.
 * The first visited tile of every row is never skipped (m_run = -inf).
 * threshold_scale_factor = 0 reproduces dense softmax attention.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers on the current CUDA device, owned
 *    by the caller, 16-byte aligned, densely packed in the layouts stated.
 *    bf16 tensors are raw IEEE bfloat16 (uint16 storage).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every device call is asynchronous on that stream and allocates no device
 *    memory.  sskip_attn_prefill_host also creates two copy streams once per
 *    device and a few events per call.  sskip_calibrate_factor and
 *    sskip_hilbert3d_order are host-only and synchronous.
 *  - The return value reports argument validation and launch errors
 *    synchronously (sskip_status).  Errors found on the device while a kernel
 *    runs (a bounded wait that ran out, an out-of-range device-side length
 *    or index) are latched in a per-device status
 *    word that sskip_get_status() reads.  No C++ exception crosses this ABI.
 *  - Outputs, the counters included, are overwritten, never accumulated.
 *  - Debug build.  libsskip_attn_debug.so exports the same functions from the
 *    same sources compiled with device-side checks of tile, ring and record
 *    indices (a stand-in for a memory checker).  A failed check latches
 *    SSKIP_ERR_DEVICE_CHECK in the status word and skips the access; a
 *    producer still completes its barrier phase, so nothing traps or hangs.
 *    Outputs are bit-identical to the release build's when no check fails.
 */
#ifndef SSKIP_ATTN_H_
#define SSKIP_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSKIP_OK = 0,
    SSKIP_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, misaligned, tsf < 0 */
    SSKIP_ERR_UNSUPPORTED = 2,  /* valid but not built: d, tile sizes, device  */
    SSKIP_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed        */
    SSKIP_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out          */
    SSKIP_ERR_DEVICE_CHECK = 5  /* a device-side index check of the debug
                                   build failed (libsskip_attn_debug.so)       */
} sskip_status;

/* Library version (major * 10000 + minor * 100 + patch). */
int sskip_version(void);

/* Human-readable name of a status code (static string; never NULL). */
const char* sskip_status_string(int status);

/* Returns SSKIP_OK when `device` is an sm_100 GPU this build runs on,
 * SSKIP_ERR_UNSUPPORTED otherwise, SSKIP_ERR_CUDA if the query failed. */
int sskip_device_supported(int device);

/*
 * Prefill: causal or non-causal Skip-Softmax attention over one sequence per
 * batch entry (the compute-bound phase of the article's "Skip Softmax 带来了
 * 哪些实战好处" section: skipping the softmax and BMM2 removes FLOPs).
 *
 *   q   [B, Hq,  L, d] bf16      o   [B, Hq, L, d] bf16 (written)
 *   k   [B, Hkv, L, d] bf16      lse [B, Hq, L] fp32, natural log of the
 *   v   [B, Hkv, L, d] bf16          row sum over the KEPT keys (written)
 *
 *   Query head hq reads kv head hq / (Hq / Hkv) (grouped-query attention).
 *   causal: key c is visible to row r iff c <= r.  Tiles wholly above the
 *   diagonal are not visited and not counted.
 *   sm_scale: logit scale (commonly 1/sqrt(d)).
 *   threshold_scale_factor >= 0: t = threshold_scale_factor / L.
 *   Br, Bc: query / key tile sizes; the skip decision is taken per Br x Bc
 *   tile of ONE query head.  Supported: (Br, Bc) in {(64, 64), (128, 128)}.
 *   d in {64, 128}.  L >= 1, Hq % Hkv == 0.
 *   skip_count: optional device uint64[2] = {skipped tiles, visited tiles}
 *   summed over the call; may be NULL.
 */
int sskip_attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int Hq, int Hkv, int L, int d, int causal, float sm_scale,
                       float threshold_scale_factor, int Br, int Bc,
                       unsigned long long* skip_count, void* stream);

/*
 * Same as sskip_attn_prefill, plus an optional per-tile record of the
 * decisions: tile_state [B, Hq, ceil(L/Br), ceil(L/Bc)] uint8 on the device,
 * 0 = not visited, 1 = kept, 2 = skipped.  NULL disables it.
 */
int sskip_attn_prefill_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int L, int d, int causal, float sm_scale,
                          float threshold_scale_factor, int Br, int Bc,
                          unsigned long long* skip_count, uint8_t* tile_state, void* stream);

/*
 * Prefill with a choice of vote granularity.  vote_rows = Br is the block
 * vote of sskip_attn_prefill.  vote_rows = 32 takes the same test per warp
 * slice of 32 query rows, the granularity of the "稀疏 Warp 在线 Softmax"
 * stage in the SpargeAttn article (its local-vs-global maximum test, taken
 * per warp): each slice of a tile passes or fails on its own rows, and a
 * slice that passes leaves its rows' m, l and O untouched (no exponentials
 * for it).  The tile's V load and its P.V still run unless every slice of
 * the tile passes, so the block decisions (and the tile_state record) equal
 * those of the block vote whenever t < 1; the outputs differ only in the
 * small terms the passing slices drop.
 *
 *   vote_rows: Br or 32; anything else is SSKIP_ERR_UNSUPPORTED.
 *   counts: optional device uint64[4] = {skipped tiles, visited tiles,
 *     skipped slices, visited slices}; a slice is counted when it holds at
 *     least one row < L.  With vote_rows = Br the slices are the tiles.
 *   tile_state: optional, as in sskip_attn_prefill_ex.
 *   slice_mask: optional device uint8 [B, Hq, ceil(L/Br), ceil(L/Bc)]:
 *     0 = tile not visited, else 0x80 | bit s set when slice s (rows
 *     [s * vote_rows, (s + 1) * vote_rows) of the query tile) skipped it.  A
 *     slice with no row < L passes vacuously (its bit is set).
 *   tile_crit: optional device fp32 [B, Hq, ceil(L/Br), ceil(L/Bc)], 4-byte
 *     aligned: per visited tile its critical value, the natural log of the
 *     smallest threshold_scale_factor that skips it under the block vote,
 *     c = max over valid rows (m_local - m_run) + ln L, with m_run the running
 *     maximum before the tile; +inf for a tile no factor skips (the first
 *     tile of a row), NaN where the tile is not visited.  While t < 1 the
 *     running maximum does not depend on what was skipped, so the record is
 *     the same at every factor below L and the call skips a tile exactly when
 *     ln(threshold_scale_factor) > c.  The input of sskip_calibrate_factor.
 */
int sskip_attn_prefill_vote(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int Hq, int Hkv, int L, int d, int causal, float sm_scale,
                            float threshold_scale_factor, int Br, int Bc, int vote_rows,
                            unsigned long long* counts, uint8_t* tile_state,
                            uint8_t* slice_mask, float* tile_crit, void* stream);

/*
 * Prefill from HOST memory to HOST memory, the copies overlapped with the
 * kernels.  Computes exactly sskip_attn_prefill_ex (no tile record) on the
 * same arguments: q_h, k_h, v_h, o_h, lse_h are host buffers in the layouts
 * above (pinned memory lets the copies overlap; pageable memory works but
 * serialises them); q_d, k_d, v_d, o_d, lse_d are device buffers of the same
 * sizes, owned by the caller (inputs are staged there; their contents after
 * the call are the staged inputs and the outputs).
 *
 * The kv heads of each batch entry are cut into groups of kv_per_chunk (0 =
 * the smallest group that fills one wave of CTAs on a 148-SM part: small
 * groups shorten the pipeline's fill and drain);
 * a group's query heads, keys, values, outputs and lse rows are contiguous,
 * and group c's host-to-device copy, group c-1's prefill and group c-2's
 * device-to-host copy run concurrently on two library-owned copy streams and
 * `stream`.  Every query tile is computed by the same kernel code as in the
 * one-shot call, so the outputs are bit-identical to it.
 * skip_count: optional device uint64[2], summed over the groups.
 * The call returns after enqueueing; the outputs are in host memory once
 * `stream` has completed (it waits for the last copy).  The two copy streams
 * are created on first use, once per device, and kept for the process's life.
 * Every argument check runs before the first copy; if an error is returned
 * after copies were enqueued, `stream` still waits for all of them, so the
 * buffers may be reused in stream order.
 */
int sskip_attn_prefill_host(const void* q_h, const void* k_h, const void* v_h, void* o_h,
                            float* lse_h, void* q_d, void* k_d, void* v_d, void* o_d, float* lse_d,
                            int B, int Hq, int Hkv, int L, int d, int causal, float sm_scale,
                            float threshold_scale_factor, int Br, int Bc, int kv_per_chunk,
                            unsigned long long* skip_count, void* stream);

/*
 * Decode: one new query token per sequence against a contiguous KV cache,
 * split over the key axis and merged by log-sum-exp (the bandwidth-bound
 * phase of the article's "Skip Softmax 带来了哪些实战好处" section: a skipped
 * block costs no V load).
 *
 *   q       [B, Hq, d] bf16               o   [B, Hq, d] bf16 (written)
 *   kcache  [B, Hkv, Lmax, d] bf16         lse [B, Hq] fp32 natural log
 *   vcache  [B, Hkv, Lmax, d] bf16             (written)
 *   seqlens [B] int32 on the device, 1 <= seqlens[b] <= Lmax; rows at or
 *           beyond seqlens[b] are never read.  The host cannot see these
 *           values, so the kernel checks them: a length outside [1, Lmax]
 *           latches SSKIP_ERR_INVALID_ARG in the device status word (read it
 *           with sskip_get_status) and is clamped into [0, Lmax] before use,
 *           so no access leaves the sequence's cache slab; a clamped length
 *           of 0 gives O = 0 and lse = -inf for that sequence's heads.
 *
 *   A decode tile is the G = Hq / Hkv query heads that share one kv head
 *   times Bc keys; the G heads take ONE joint decision, so a skipped tile
 *   really loads no V bytes.  t_b = threshold_scale_factor / seqlens[b].
 *   The key tiles of each (b, kv head) are cut into num_splits contiguous
 *   chunks of c = ceil(n_k / num_splits) tiles (n_k = ceil(seqlens[b] / Bc));
 *   each chunk runs its own online softmax from m_run = -inf, and the chunks
 *   merge by log-sum-exp.
 *   Supported: d in {64, 128}, Bc = 64, G in {1, 2, 4, 8}, 1 <= num_splits <= 64.
 *   workspace: device scratch of at least
 *   sskip_attn_decode_workspace_size(B, Hq, d, num_splits) bytes, 256-byte
 *   aligned, owned by the caller; its contents need no initialisation and
 *   are meaningless after the call.
 *   skip_count: optional device uint64[2] = {skipped, visited} decode tiles.
 */
size_t sskip_attn_decode_workspace_size(int B, int Hq, int d, int num_splits);

int sskip_attn_decode(const void* q, const void* kcache, const void* vcache,
                      const int* seqlens, void* o, float* lse,
                      int B, int Hq, int Hkv, int Lmax, int d, float sm_scale,
                      float threshold_scale_factor, int Bc, int num_splits,
                      void* workspace, size_t workspace_bytes,
                      unsigned long long* skip_count, void* stream);

/* Same as sskip_attn_decode, plus tile_state [B, Hkv, ceil(Lmax/Bc)] uint8
 * (0 = not visited, 1 = kept, 2 = skipped); NULL disables it. */
int sskip_attn_decode_ex(const void* q, const void* kcache, const void* vcache,
                         const int* seqlens, void* o, float* lse,
                         int B, int Hq, int Hkv, int Lmax, int d, float sm_scale,
                         float threshold_scale_factor, int Bc, int num_splits,
                         void* workspace, size_t workspace_bytes,
                         unsigned long long* skip_count, uint8_t* tile_state, void* stream);

/*
 * Same as sskip_attn_decode_ex, plus an optional record of each decode tile's
 * critical value (see sskip_attn_prefill_vote): tile_crit, device fp32
 * [B, Hkv, ceil(Lmax/Bc)], 4-byte aligned; c = max over the G heads of
 * (m_local - m_run) + ln(seqlens[b]) with m_run the running maximum of the
 * tile's split (+inf for the first tile of a split), NaN for tiles past
 * seqlens[b].  The call skips a tile exactly when ln(factor) > c while
 * factor < seqlens[b].
 */
int sskip_attn_decode_crit(const void* q, const void* kcache, const void* vcache,
                           const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                           int Lmax, int d, float sm_scale, float threshold_scale_factor, int Bc,
                           int num_splits, void* workspace, size_t workspace_bytes,
                           unsigned long long* skip_count, uint8_t* tile_state, float* tile_crit,
                           void* stream);

/*
 * Threshold calibration (the Model Optimizer tutorial's step 4 and the
 * TensorRT-LLM article's closing "target sparsity in, threshold out" goal):
 * pick the threshold_scale_factor that skips target_ratio of the visited
 * tiles, from a tile_crit record taken on calibration inputs.  HOST memory:
 * tile_crit is a host copy of the record (n floats, NaN = not visited).
 *
 *   k = ceil(target_ratio * visited) tiles must be skipped; the factor is
 *   placed halfway, in natural log, between the k-th smallest critical value
 *   and the next larger one (capped by max_factor), so every tile whose
 *   critical value is at most the k-th is skipped and no other.
 *   max_factor: the smallest context length of the data (the factor must keep
 *     t = factor / L < 1 for the record to hold); <= 0 disables the cap.
 *   factor (out): the factor; 0 when target_ratio rounds to zero tiles.
 *   achieved_ratio (out, may be NULL): skipped / visited at that factor
 *     (>= target_ratio; above it only when critical values tie).
 *   visited_out (out, may be NULL): the number of visited tiles.
 *   Returns SSKIP_ERR_UNSUPPORTED when the target cannot be reached below
 *   max_factor, SSKIP_ERR_INVALID_ARG for a bad argument or an empty record.
 *   Pure host code: no CUDA call.
 */
int sskip_calibrate_factor(const float* tile_crit, size_t n, double target_ratio,
                           double max_factor, double* factor, double* achieved_ratio,
                           long long* visited_out);

/*
 * Decode for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is a deployment variant of sskip_attn_decode.
 *
 * Who needs it: code that must not call cudaMalloc -- embedded runtimes
 * without a device allocator, plugins whose host framework owns every device
 * allocation, latency-critical serving loops that forbid allocation after
 * start-up.  The split-KV
 * decode needs scratch for its per-split partial results; here that scratch is
 * one fixed device array inside this library of
 * SSKIP_DECODE_NOALLOC_SCRATCH_BYTES (32 MiB), reserved on every GPU that loads
 * the library until the process exits.  The caller still passes inputs and
 * outputs exactly as for sskip_attn_decode; everything else is the same.
 *
 *  - Returns SSKIP_ERR_UNSUPPORTED when the call would need more scratch than
 *    the array holds, i.e. when
 *    sskip_attn_decode_workspace_size(B, Hq, d, num_splits) exceeds
 *    SSKIP_DECODE_NOALLOC_SCRATCH_BYTES (for example B = 64, Hq = 32, d = 128,
 *    16 splits needs 16.9 MB and fits).
 *  - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture begins.
 *  - Every call shares the one array, which keeps the last call's contents
 *    (the kernels overwrite all of it they read).  Calls that overlap on the
 *    GPU -- on different streams, or from different threads -- race on it and
 *    give undefined results: serialise them.
 */
#define SSKIP_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)

int sskip_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                              const int* seqlens, void* o, float* lse,
                              int B, int Hq, int Hkv, int Lmax, int d, float sm_scale,
                              float threshold_scale_factor, int Bc, int num_splits,
                              unsigned long long* skip_count, void* stream);

/*
 * Decode with the per-step tensors in HOST memory: q_h [B, Hq, d] bf16 and
 * seqlens_h [B] int32 are copied to the caller's device buffers q_d and
 * seqlens_d, the decode runs exactly as sskip_attn_decode_ex (no tile record)
 * against the device-resident kcache / vcache, and o_d / lse_d are copied
 * back to o_h [B, Hq, d] bf16 and lse_h [B, Hq] fp32, all in order on
 * `stream` (the step's copies are a few hundred KB: nothing to overlap).
 * Pinned host memory keeps the copies asynchronous.  Validation as in
 * sskip_attn_decode_ex.
 */
int sskip_attn_decode_host(const void* q_h, const int* seqlens_h, void* o_h, float* lse_h,
                           void* q_d, int* seqlens_d, void* o_d, float* lse_d,
                           const void* kcache, const void* vcache, int B, int Hq, int Hkv,
                           int Lmax, int d, float sm_scale, float threshold_scale_factor, int Bc,
                           int num_splits, void* workspace, size_t workspace_bytes,
                           unsigned long long* skip_count, void* stream);

/*
 * One serving step of one attention layer with a factor per phase: the
 * TensorRT-LLM article ("实战演练") lets threshold_scale_factor be a single
 * number or a {prefill: 1000, decode: 500} pair, each divided by its own
 * context length.  The step runs, in this order on `stream`:
 *   - the prefill of Bp whole sequences of length L (skipped when Bp = 0),
 *     exactly sskip_attn_prefill_ex(q, k, v, o, lse, Bp, Hq, Hkv, L, d, causal,
 *     sm_scale, tsf_prefill, Br, Bc, prefill_count, NULL, stream), so
 *     t = tsf_prefill / L;
 *   - the decode of Bd sequences against their caches (skipped when Bd = 0),
 *     exactly sskip_attn_decode_ex(dq, kcache, vcache, seqlens, dout, dlse, Bd,
 *     Hq, Hkv, Lmax, d, sm_scale, tsf_decode, 64, num_splits, workspace,
 *     workspace_bytes, decode_count, NULL, stream), so t_b = tsf_decode /
 *     seqlens[b].
 * Hq, Hkv, d and sm_scale are the layer's and shared by both phases.  Returns
 * the first failing status (the decode is not enqueued after a prefill
 * error).  Bp = Bd = 0 is SSKIP_ERR_INVALID_ARG.
 */
int sskip_attn_step(const void* q, const void* k, const void* v, void* o, float* lse, int Bp,
                    int L, int causal, int Br, int Bc, unsigned long long* prefill_count,
                    const void* dq, const void* kcache, const void* vcache, const int* seqlens,
                    void* dout, float* dlse, int Bd, int Lmax, int num_splits, void* workspace,
                    size_t workspace_bytes, unsigned long long* decode_count, int Hq, int Hkv,
                    int d, float sm_scale, float tsf_prefill, float tsf_decode, void* stream);

/*
 * Token reordering along a 3-D Hilbert curve (SpargeAttn article, "Hilbert
 * 曲线置换": the T x H x W visual tokens are laid out along a Hilbert curve
 * before attention so that the tokens of one tile form a compact 3-D region,
 * which raises the share of tiles that can be skipped).
 *
 * sskip_hilbert3d_order: HOST call, no CUDA.  For the first L tokens of the
 * t-major raster of a T x H x W grid (token i at t = i / (H W),
 * h = (i / W) % H, w = i % W), writes perm[s] (host int32 [L]) = the raster
 * index of the token at position s of the Hilbert order: tokens sorted by
 * their position on the Hilbert curve of the smallest 2^b cube holding the
 * grid (John Skilling's index; points outside the grid are absent).
 * Requires L <= T H W.
 */
int sskip_hilbert3d_order(int T, int H, int W, int L, int32_t* perm);

/*
 * sskip_permute_rows: reorders whole rows of n_mats consecutive [L, row]
 * matrices (device memory, row = row_bytes bytes, a multiple of 4):
 *   scatter = 0 (gather):  dst[m, i, :] = src[m, idx[i], :]
 *   scatter = 1 (inverse): dst[m, idx[i], :] = src[m, i, :]
 * idx: device int32 [L], a permutation of 0 .. L-1; an index outside it is
 * latched as SSKIP_ERR_INVALID_ARG in the device status word and that row is
 * not touched.  src and dst must not overlap.  16-byte rows use 16-byte
 * accesses (pointers then 16-byte aligned), others 4-byte ones.  With perm
 * from sskip_hilbert3d_order: gather Q, K, V [B, H, L, d] into Hilbert order
 * (n_mats = B H), run a non-causal prefill, scatter O and lse back.
 */
int sskip_permute_rows(const void* src, void* dst, const int32_t* idx, long long n_mats, int L,
                       int row_bytes, int scatter, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word: SSKIP_OK, or the first device-side error latched since the last call
 * (SSKIP_ERR_TIMEOUT when a bounded wait inside a kernel ran out: the kernel
 * then abandoned its work, waited out its own copies in flight and left its
 * outputs undefined; SSKIP_ERR_INVALID_ARG when a decode length or a permute
 * index held in device memory was out of range).  Returns SSKIP_ERR_CUDA if
 * the synchronisation itself failed.
 */
int sskip_get_status(void* stream);

/*
 * Self-test of the bounded-wait watchdog: launches one tiny kernel that waits
 * on an mbarrier that nothing ever completes, with a wait limit of
 * `limit_us` microseconds (1 .. 2,000,000).  The wait runs out, the kernel
 * latches SSKIP_ERR_TIMEOUT in the status word and returns; the context stays
 * usable.  Read the result with sskip_get_status().
 */
int sskip_selftest_watchdog(unsigned int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSKIP_ATTN_H_ */
