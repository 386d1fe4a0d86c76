// prefill_sm100.cuh -- Skip-Softmax tiled attention prefill for sm_100a.
//
// The FlashAttention carrier of the TensorRT-LLM Skip-Softmax article
// ("Skip Softmax 到底怎么回事" section: logits, then softmax, then x V), with
// the block test of its "Skip Softmax 的三步走算法" section inserted between
// the two contractions: a key tile whose rows all sit more than ln(1/t) below
// their running maximum skips its softmax, its P.V (BMM2) and its V load.
//
// One CTA owns 256 query rows of one (batch, query head) as two 128-row MMA
// tiles, A and B, each with its own softmax warpgroup, so that the tensor
// core always has one tile's QK^T or P.V to run while the other tile's
// softmax works (ping-pong).  A 128-row MMA tile is one Br = 128 query tile,
// or two stacked Br = 64 query tiles that vote separately.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q_A and Q_B once, then K tiles through an
//               NK-stage ring (K is needed for every visited tile).
//   warp 1      TMEM allocator; one thread issues every tcgen05.mma:
//               per key tile j: P_A.V_j, S_A(j+1), P_B.V_j, S_B(j+1).
//   warp 2      collector: reads both warpgroups' votes on tile j, issues
//               the V_j TMA on the first "keep" (a tile both skip never
//               loads V) and writes the tile records and counts.
//   warps 4..7  softmax of tile A, thread r = TMEM lane r = query row r.
//   warps 8..11 softmax of tile B.
// A softmax warp, per key tile: loads its S rows from TMEM, masks them, takes
// the row maxima and its vote flag (do all its rows pass?), and posts it.
// The tile is skipped iff every valid row of a Br-row query tile passes; a
// warp with a row that did not pass knows the tile is kept without waiting
// for the others.  For a kept tile it computes P = exp2(S - m) in fp32,
// packs it to bf16 in place of S in TMEM, and releases the tile to the MMA
// thread, which runs O += P V with P read straight from TMEM.
// Skipped tiles cost one QK^T MMA and one row max: no exp, no P, no V bytes.
//
// Exponent reference: the vote always uses the exact running max m_run; the
// exponentials use a reference m_ref raised only when m_run exceeds it by
// more than 8 (log2 units), so O in TMEM is rescaled rarely.  O, l and the
// result O / l, lse = ln 2 * (m_ref + log2 l) do not depend on that choice.
// O needs no extra wait before a rescale: S_A(j) is issued after P_A.V_{j-1}
// and tcgen05 MMAs complete in order, so when S_A(j) is visible so is O_A.
#pragma once

#include "skip_rule.cuh"
#include "sm100_ptx.cuh"
#include "sm100_tmem.cuh"

namespace sskip {

struct PrefillParams {
  __nv_bfloat16* o;            // [B, Hq, L, D]
  float* lse;                  // [B, Hq, L]
  unsigned long long* counts;  // {skipped, visited[, slices skipped, slices visited]} or null
  uint8_t* tile_state;         // [B, Hq, n_q, n_k] or null
  uint8_t* slice_mask;         // [B, Hq, n_q, n_k] or null: 0x80 | slices that skipped
  float* tile_crit;            // [B, Hq, n_q, n_k] or null: ln of the skipping factor
  float ln_L;                  // ln(L)
  int slice_vote;              // 1: each 32-row warp slice votes alone
  int n_counts;                // 2 or 4 entries in counts
  int B, Hq, Hkv, L, G;
  int n_q;                     // ceil(L / Br)
  int n_k;                     // ceil(L / Bc)
  int n_units;                 // ceil(L / 256): 256-row units per head
  float scale_log2;            // sm_scale * log2(e)
  float log2_t;                // log2(tsf / L), -inf when tsf == 0
  int t_positive;
};

constexpr int kPfThreads = 384;
constexpr int kPfUnitRows = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kPfVoteSlots = 4;

// Tuning switches of the softmax inner loop (compile-time).
#ifndef SSKIP_PF_FMA_EXP
#define SSKIP_PF_FMA_EXP 0   // element pairs per 8 whose exp2 runs on the FMA pipe
#endif
#ifndef SSKIP_PF_RELOAD
#define SSKIP_PF_RELOAD 0     // 1, d = 128: re-read S's second half from TMEM for the exponentials (0: hold all of S)
#endif
#ifndef SSKIP_PF_RELOAD_D64
#define SSKIP_PF_RELOAD_D64 0  // at d = 64 S stays in registers from the max pass
#endif
template <int D>
__device__ __forceinline__ constexpr bool kReload() {
  return (D == 64 ? SSKIP_PF_RELOAD_D64 : SSKIP_PF_RELOAD) != 0;
}
#ifndef SSKIP_PF_NACC
#define SSKIP_PF_NACC 4       // independent packed accumulators of the row sum
#endif
#ifndef SSKIP_PF_ROUNDED_L
#define SSKIP_PF_ROUNDED_L 0  // 1: O is divided by the sum of the bf16 P that P.V used
#endif
#ifndef SSKIP_PF_EXT_RELOAD
#define SSKIP_PF_EXT_RELOAD 0  // 1: the per-warp-vote build re-reads S at every d
#endif
#ifndef SSKIP_PF_PRODUCER_REGS
#define SSKIP_PF_PRODUCER_REGS 88  // registers of the producer, MMA and collector warps (<= 88 with 208)
#endif
#ifndef SSKIP_PF_FMA_EXP_D64
#define SSKIP_PF_FMA_EXP_D64 SSKIP_PF_FMA_EXP  // the same, for head dim 64
#endif
// At d = 64 a tile's exponentials outweigh its MMAs (16 exp2 per clock per SM
// on MUFU against 128 x 128 x 64 x 4 FLOP), so part of them may run on the FMA
// pipe instead; at d = 128 the two are balanced.
template <int D>
__device__ __forceinline__ constexpr bool exp2_on_fma(int pair) {
  constexpr int n = D == 64 ? SSKIP_PF_FMA_EXP_D64 : SSKIP_PF_FMA_EXP;
  return n > 0 && ((pair & 7) * n) % 8 < n;
}
constexpr float kPackBias = 0.0f;

template <int D, int BC>
struct PrefillCfg {
  static constexpr bool kBig = (D * BC >= 128 * 128);
  static constexpr int kNK = kBig ? 3 : 4;  // K stages
  static constexpr int kNV = kBig ? 2 : 3;  // V stages
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = BC * D * 2;
  static constexpr int kQ = 0;  // Q_A, then Q_B
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kNK * kKVBytes;
  static constexpr int kBar = kV + kNV * kKVBytes;
  // One S/P buffer of Bc columns per query tile, then O_A and O_B.
  static constexpr int kOCol = 2 * BC;  // first TMEM column of O_A (O_B follows)
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], then per
  // warpgroup s_full, p_lo, p_hi, then vote[2][VS], vote_read[2][VS], mma_done
  static constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 3 * 2 + 4 * kPfVoteSlots + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  // warp vote flags [2 wg][VS][4], warp gaps [2 wg][VS][4] (fp32), tmem, abort
  static constexpr int kMiscInts = 16 * kPfVoteSlots + 2;
  static constexpr int kTotal = kMisc + kMiscInts * 4;
  static constexpr int kAlloc = kTotal + 1024;  // room to align the base to 1 KB
  static constexpr int kTmemCols = (kOCol + 2 * D) <= 256 ? 256 : 512;
  static_assert(kQBytes % 1024 == 0 && kKVBytes % 1024 == 0, "tiles keep 1 KB alignment");
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

// EXT = false compiles the plain block vote with the tile_state record only;
// EXT = true adds the per-warp vote, the slice and critical-value records and
// the four counters (kept out of the plain kernel, which they slow down).
//
// A kept tile's P (bf16) is stored over the first Bc/2 of its S columns in
// two halves of Bc/2 keys, and P.V runs as two matching halves:
//   O += P_lo(j) V_j[:Bc/2]   as soon as P of the first half is stored;
//   O += P_hi(j) V_j[Bc/2:]   once all of P is stored.
// With one S buffer per query tile, S(j+1) = Q K_{j+1}^T then goes to the
// same columns: tcgen05 MMAs of one thread complete in issue order, so S(j+1)
// never overwrites a P that P.V still reads, and its commit makes S(j+1) and
// O visible together.  A skipped tile releases its S columns at the vote and
// the next S follows at once.
template <int D, int BR, int BC, bool CAUSAL, bool EXT>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D, BC>;
  constexpr int NK = C::kNK, NV = C::kNV, VS = kPfVoteSlots;
  constexpr int NGRP = 128 / BR;  // vote groups per 128-row MMA tile
  constexpr int WPG = BR / 32;    // warps per vote group
  constexpr int HK = BC / 2;      // keys per half tile
  constexpr int HP = HK / 2;      // packed bf16 P columns per half tile
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BC, 0, 0);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
  static_assert(BR == 64 || BR == 128, "Br");
  static_assert(BC == 64 || BC == 128, "Bc");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  int* misc = reinterpret_cast<int*>(smem + C::kMisc);
  // Warp vote flags [2 wg][VS][4 warps]: 1 when every row of the warp passes.
  volatile int* wflag = misc;
  volatile float* wgap = reinterpret_cast<volatile float*>(misc + 8 * VS);  // [2 wg][VS][4 warps]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 16 * VS);
  volatile int* abort_flag = misc + 16 * VS + 1;
  // First flag (and gap) of warpgroup w's vote on key tile j.
  auto vslot = [&](int w, int j) { return (w * VS + j % VS) * 4; };

  const uint32_t b_qfull = smem_u32(&bars[0]);
  auto b_kfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_kempty = [&](int s) { return smem_u32(&bars[1 + NK + s]); };
  auto b_vfull = [&](int s) { return smem_u32(&bars[1 + 2 * NK + s]); };
  auto b_vempty = [&](int s) { return smem_u32(&bars[1 + 2 * NK + NV + s]); };
  constexpr int kWgBar = 1 + 2 * NK + 2 * NV;
  // Signals between a query tile's softmax and the MMA thread.  With one S
  // buffer per query tile neither side can run a phase ahead of the other.
  //   s_full  S(w, j) is in TMEM                 (MMA -> softmax; parity j)
  //   p_lo    P of the first Bc/2 keys stored, or the tile skipped
  //                                              (softmax -> MMA; parity j)
  //   p_hi    all of P stored                    (softmax -> MMA, kept tile k)
  auto b_sfull = [&](int w) { return smem_u32(&bars[kWgBar + w]); };
  auto b_plo = [&](int w) { return smem_u32(&bars[kWgBar + 2 + w]); };
  auto b_phi = [&](int w) { return smem_u32(&bars[kWgBar + 4 + w]); };
  // The vote on key tile j: each softmax warp stores its flag (and gap) in
  // slot j % VS and arrives; the collector warp and the softmax warps whose
  // own rows all passed read the four flags once the phase is complete (the
  // MMA thread reads them after p_lo).  vote_read: the collector has read the
  // slot, which may then take tile j + VS.
  auto b_vote = [&](int w, int j) { return smem_u32(&bars[kWgBar + 6 + w * VS + j % VS]); };
  auto b_vread = [&](int w, int j) {
    return smem_u32(&bars[kWgBar + 6 + 2 * VS + w * VS + j % VS]);
  };
  auto vote_par = [&](int j) { return uint32_t((j / VS) & 1); };
  const uint32_t b_mmadone = smem_u32(&bars[kWgBar + 6 + 4 * VS]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: 256 rows of one (batch, query head).  CTAs are ordered by
  // (batch, kv head), then unit (heaviest causal unit first), then the kv
  // head's G query heads: the CTAs resident at any time mostly read one kv
  // head's K and V, which then stay in L2 instead of being re-read from HBM
  // by every unit of every head.
  const int per_grp = p.n_units * p.G;
  const int grp = blockIdx.x / per_grp;
  const int rem = blockIdx.x - grp * per_grp;
  const int ublk = rem / p.G;
  const int iu = CAUSAL ? (p.n_units - 1 - ublk) : ublk;
  const int b = grp / p.Hkv, kvh = grp % p.Hkv;
  const int hq = kvh * p.G + (rem - ublk * p.G);
  const int row0 = iu * kPfUnitRows;

  // Key tiles each MMA tile visits (the union over its vote groups).
  auto tiles_visited = [&](int w) {
    int n = 0;
#pragma unroll
    for (int g = 0; g < NGRP; ++g) {
      const int it = (row0 + 128 * w) / BR + g;
      if (it < p.n_q) {
        const int jm = CAUSAL ? min(p.n_k - 1, ((it + 1) * BR - 1) / BC) : p.n_k - 1;
        n = max(n, jm + 1);
      }
    }
    return n;
  };
  const int n_a = tiles_visited(0), n_b = tiles_visited(1);
  const int n_j = max(n_a, n_b);
  // (Every thread computes the same unit, so all return together, before
  // any barrier.)
  if (!dev_check(b < p.B && hq < p.Hq && kvh < p.Hkv && iu < p.n_units && row0 < p.L &&
                 n_j <= p.n_k))
    return;
  static_assert(C::kOCol + 2 * D <= C::kTmemCols, "TMEM columns");

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    for (int s = 0; s < NK; ++s) { mbar_init(b_kfull(s), 1); mbar_init(b_kempty(s), 1); }
    for (int s = 0; s < NV; ++s) { mbar_init(b_vfull(s), 1); mbar_init(b_vempty(s), 1); }
    for (int w = 0; w < 2; ++w) {
      mbar_init(b_sfull(w), 1);
      mbar_init(b_plo(w), 4);  // one arrival per softmax warp
      mbar_init(b_phi(w), 4);
    }
    for (int w = 0; w < 2; ++w)
      for (int s = 0; s < VS; ++s) { mbar_init(b_vote(w, s), 4); mbar_init(b_vread(w, s), 1); }
    mbar_init(b_mmadone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    regs_dealloc<SSKIP_PF_PRODUCER_REGS>();
    if (warp == 0 && lane == 0) {
      // ================= TMA producer: Q_A, Q_B, then the K ring ==========
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      mbar_arrive_expect_tx(b_qfull, 2 * C::kQBytes);
#pragma unroll
      for (int w = 0; w < 2; ++w)
#pragma unroll
        for (int blk = 0; blk < D / 64; ++blk)
          tma_load_3d(sbase + C::kQ + w * C::kQBytes + blk * 128 * 128, &tmQ, b_qfull, blk * 64,
                      row0 + 128 * w, b * p.Hq + hq);
      int last = -1;
      const int n_w[2] = {n_a, n_b};
      for (int j = 0; j < n_j; ++j) {
        const int s = j % NK;
        if (j >= NK && !mbar_wait(b_kempty(s), ((j / NK) - 1) & 1, abort_flag)) break;
        // No vote on tile j (which needs K_j) before the collector has read
        // the same slots' votes on tile j - VS.
        if (j >= VS) {
          bool okv = true;
#pragma unroll
          for (int w = 0; w < 2; ++w)
            if (okv && j - VS < n_w[w]) okv = mbar_wait(b_vread(w, j), vote_par(j) ^ 1u, abort_flag);
          if (!okv) break;
        }
        if (!dev_check(j < p.n_k && b * p.Hkv + kvh < p.B * p.Hkv)) {
          mbar_arrive(b_kfull(s));  // the phase completes without data
          continue;
        }
        mbar_arrive_expect_tx(b_kfull(s), C::kKVBytes);
#pragma unroll
        for (int blk = 0; blk < D / 64; ++blk)
          tma_load_3d(sbase + C::kK + s * C::kKVBytes + blk * BC * 128, &tmK, b_kfull(s),
                      blk * 64, j * BC, b * p.Hkv + kvh);
        last = j;
      }
      if (*abort_flag) {  // leave no copy in flight
        int dummy = 0;
        for (int j = max(0, last - NK + 1); j <= last; ++j)
          mbar_wait(b_kfull(j % NK), (j / NK) & 1, &dummy);
        mbar_wait(b_qfull, 0, &dummy);
      }
    } else if (warp == 1 && lane == 0) {
      // ================= MMA issuer =================
      // Descriptors are built once per operand; a K step only moves the start
      // address field (bits 0-13, in 16-byte units), which never carries out
      // of it since shared addresses stay below 256 KB.
      const uint64_t dq0 = smem_desc_sw128(sbase + C::kQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + C::kK, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sbase + C::kV, BC * 128, 1024);
      // S = Q_w K_j^T into query tile w's TMEM columns [w Bc, w Bc + Bc).
      auto issue_s = [&](int w, int j) {
        const uint64_t da = dq0 + (uint64_t)((w * C::kQBytes) >> 4);
        const uint64_t db = dk0 + (uint64_t)(((j % NK) * C::kKVBytes) >> 4);
        const uint32_t d_tmem = tmem + w * BC;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = ((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * (BC * 128) + (kk & 3) * 32) >> 4;
          umma_ss(d_tmem, da + oa, db + ob, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      int pv_count[2] = {0, 0};
      // O(w) += P[:, half h] V[half h], P read from query tile w's S/P
      // columns, V from slot vs.
      auto issue_pv_half = [&](int w, int vs, int h) {
        const uint32_t p_tmem = tmem + w * BC;
        const uint32_t o_tmem = tmem + C::kOCol + w * D;
        const uint64_t dv = dv0 + (uint64_t)((vs * C::kKVBytes) >> 4);
#pragma unroll
        for (int k2 = 0; k2 < HK / 16; ++k2) {
          const int kk = h * (HK / 16) + k2;
          const uint32_t acc = (kk > 0 || pv_count[w] > 0) ? 1u : 0u;
          umma_ts(o_tmem, p_tmem + kk * 8, dv + (uint64_t)((kk * 16 * 128) >> 4), IDESC_PV, acc);
        }
        if (h == 1) ++pv_count[w];
      };
      const int n_w[2] = {n_a, n_b};
      int kc_w[2] = {0, 0};  // kept tiles per warpgroup (phase of p_lo / p_hi)
      int kc = 0;            // tiles some warpgroup kept: the V load number
      bool ok = mbar_wait(b_qfull, 0, abort_flag);
      // Key tile j, warpgroup A then B: its decision; for a kept tile P_lo V
      // as soon as P_lo is stored and P_hi V once P is complete; then S(j+1),
      // which overwrites the P(j) that P.V just read.  V_j is in slot kc % NV
      // (the collector's numbering).
      if (ok && n_j > 0) {
        ok = mbar_wait(b_kfull(0), 0, abort_flag);
        tc_fence_after();
        if (ok) {
#pragma unroll
          for (int w = 0; w < 2; ++w)
            if (n_w[w] > 0) {
              issue_s(w, 0);
              umma_commit(b_sfull(w));
            }
          umma_commit(b_kempty(0));
        }
      }
      for (int j = 0; ok && j < n_j; ++j) {
        const int vs = kc % NV;
        bool any_kept = false, v_ready = false, k_ready = false;
        // K_{j+1} is waited for just before its first use, so that a late
        // K tile never holds back a P.V.
        auto need_k = [&]() {
          if (!k_ready) k_ready = mbar_wait(b_kfull((j + 1) % NK), ((j + 1) / NK) & 1, abort_flag);
          return k_ready;
        };
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (j >= n_w[w]) continue;
          const bool s_next = j + 1 < n_w[w];
          // Every visited tile completes one p_lo phase (a skipped one at its
          // decision); the four flags are stored before it.
          if (!mbar_wait(b_plo(w), j & 1, abort_flag)) { ok = false; break; }
          const volatile int* f = wflag + vslot(w, j);
          if (!(f[0] & f[1] & f[2] & f[3])) {
            any_kept = true;
            const uint32_t par = kc_w[w] & 1;
            if (!v_ready) {
              if (!mbar_wait(b_vfull(vs), (kc / NV) & 1, abort_flag)) { ok = false; break; }
              v_ready = true;
            }
            tc_fence_after();
            issue_pv_half(w, vs, 0);
            if (!mbar_wait(b_phi(w), par, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_pv_half(w, vs, 1);
            ++kc_w[w];
            if (s_next) {
              if (!need_k()) { ok = false; break; }
              issue_s(w, j + 1);
            }
          } else if (s_next) {
            if (!need_k()) { ok = false; break; }
            tc_fence_after();
            issue_s(w, j + 1);
          }
          if (s_next) umma_commit(b_sfull(w));
        }
        if (!ok) break;
        if (any_kept) {
          umma_commit(b_vempty(vs));
          ++kc;
        }
        if (j + 1 < n_j) umma_commit(b_kempty((j + 1) % NK));
      }
      // Every MMA issued by this thread completes before the epilogue reads O
      // and before TMEM is released.
      umma_commit(b_mmadone);
      int no_abort = 0;
      mbar_wait(b_mmadone, 0, &no_abort);
    } else if (warp == 2 && lane == 0) {
      // ================= collector: reads the votes, issues V, records =====
      // Both query tiles' votes on tile j, in tile order.  The first "keep"
      // starts the V_j load, so its latency hides behind that warpgroup's
      // exponentials.  Loads are numbered in tile order over the tiles some
      // warpgroup kept and go to slot number % NV; a tile both skip costs
      // nothing here.  The tile records and the counts are written here too,
      // off the softmax warps' path.
      tma_prefetch_desc(&tmV);
      const int n_w[2] = {n_a, n_b};
      int kc = 0, last = -1;
      long long n_vis = 0, n_skip = 0;
      for (int j = 0; j < n_j && !*abort_flag; ++j) {
        bool issued = false;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (j >= n_w[w]) continue;
          if (!mbar_wait(b_vote(w, j), vote_par(j), abort_flag)) break;
          const int fs = vslot(w, j);
          int fl[4];
          float gm[NGRP];
#pragma unroll
          for (int q = 0; q < 4; ++q) fl[q] = wflag[fs + q];
#pragma unroll
          for (int g = 0; g < NGRP; ++g) {
            gm[g] = -INFINITY;
            if (EXT && p.tile_crit)
#pragma unroll
              for (int q = 0; q < WPG; ++q) gm[g] = fmaxf(gm[g], wgap[fs + g * WPG + q]);
          }
          mbar_arrive(b_vread(w, j));  // the slot may now take tile j + VS
          bool kept = false;
#pragma unroll
          for (int g = 0; g < NGRP; ++g) {
            bool all = true;
            uint32_t bits = 0;
#pragma unroll
            for (int q = 0; q < WPG; ++q) {
              all = all && fl[g * WPG + q] != 0;
              bits |= fl[g * WPG + q] != 0 ? (1u << q) : 0u;
            }
            const int it = (row0 + 128 * w) / BR + g;  // this group's query tile
            if (it >= p.n_q) continue;
            const int jm = CAUSAL ? min(p.n_k - 1, ((it + 1) * BR - 1) / BC) : p.n_k - 1;
            if (j > jm) continue;  // the group does not visit tile j
            kept = kept || !all;
            const size_t rec = (((size_t)b * p.Hq + hq) * p.n_q + it) * p.n_k + j;
            if (!dev_check(j < p.n_k && rec < (size_t)p.B * p.Hq * p.n_q * p.n_k)) continue;
            ++n_vis;
            n_skip += all ? 1 : 0;
            if (p.tile_state) p.tile_state[rec] = all ? 2 : 1;
            if (EXT && p.slice_mask)
              p.slice_mask[rec] = uint8_t(0x80u | (p.slice_vote ? bits : (all ? 1u : 0u)));
            // Skipped iff ln(tsf) > max gap * ln 2 + ln L (for every factor below L).
            if (EXT && p.tile_crit) p.tile_crit[rec] = gm[g] * 0.69314718055994531f + p.ln_L;
          }
          if (kept && !issued) {
            const int vs = kc % NV;
            if (kc >= NV && !mbar_wait(b_vempty(vs), ((kc / NV) - 1) & 1, abort_flag)) break;
            if (!dev_check(j < p.n_k && vs < NV)) {
              mbar_arrive(b_vfull(vs));  // the phase completes without data
            } else {
              mbar_arrive_expect_tx(b_vfull(vs), C::kKVBytes);
#pragma unroll
              for (int blk = 0; blk < D / 64; ++blk)
                tma_load_3d(sbase + C::kV + vs * C::kKVBytes + blk * BC * 128, &tmV, b_vfull(vs),
                            blk * 64, j * BC, b * p.Hkv + kvh);
            }
            issued = true;
            last = kc++;
          }
        }
      }
      if (*abort_flag) {
        int dummy = 0;
        for (int k = max(0, last - NV + 1); k <= last; ++k)
          mbar_wait(b_vfull(k % NV), (k / NV) & 1, &dummy);
      }
      if (p.counts) {
        atomicAdd(&p.counts[0], (unsigned long long)n_skip);
        atomicAdd(&p.counts[1], (unsigned long long)n_vis);
        if (EXT && p.n_counts == 4 && !p.slice_vote) {  // one slice per block
          atomicAdd(&p.counts[2], (unsigned long long)n_skip);
          atomicAdd(&p.counts[3], (unsigned long long)n_vis);
        }
      }
    }
  } else {
    regs_alloc<208>();
    // ================= softmax warpgroups =================
    const int wg = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int wq = warp & 3;         // TMEM lane quadrant
    const int r = wq * 32 + lane;    // row within the 128-row tile
    const int grp = r / BR;
    const int row = row0 + 128 * wg + r;
    const bool row_in = row < p.L;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t tO = tmem + C::kOCol + wg * D + lane_base;
    const int n_own = wg == 0 ? n_a : n_b;
    // Last key tile this row's vote group visits (-1: the group is padding).
    const int my_tile = (row0 + 128 * wg) / BR + grp;
    const int my_jmax = my_tile >= p.n_q ? -1
                        : CAUSAL ? min(p.n_k - 1, ((my_tile + 1) * BR - 1) / BC) : p.n_k - 1;
    const float log2_t = p.log2_t;
    const bool t_pos = p.t_positive != 0;
    const float scale = p.scale_log2;

    // l_run sums P in fp32 (for lse); lr_run sums the bf16-rounded P that the
    // P.V MMA applied, so that O / lr_run weighs V with weights summing to 1.
    float m_run = -INFINITY, m_ref = -INFINITY, l_run = 0.f, lr_run = 0.f;
    long long n_svis = 0, n_sskip = 0;

    // This warp's part of a signal counted once per softmax warp: its TMEM
    // accesses are complete (the caller waited for them) and ordered before
    // the MMA warp's next tcgen05 operation.
    auto warp_signal = [&](uint32_t bar) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    for (int j = 0; j < n_j; ++j) {
      if (j >= n_own) break;  // no row of this query tile visits tile j or later
      const uint32_t tS = tmem + wg * BC + lane_base;
      mbar_wait(b_sfull(wg), j & 1, abort_flag);
      tc_fence_after();
      __syncwarp();
      uint32_t sr[BC];
#pragma unroll
      for (int c = 0; c < BC / 32; ++c) tmem_ld32_async(tS + c * 32, sr + c * 32);
      if constexpr (BC == 128) tmem_wait_ld_tie128(sr);
      else tmem_wait_ld_tie64(sr);
      float* s = reinterpret_cast<float*>(sr);

      // Mask: keys past L, and keys after the row in causal attention.
      const int key0 = j * BC;
      const bool need_mask = (key0 + BC > p.L) || (CAUSAL && key0 + BC - 1 > row);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BC; ++c) {
          const int key = key0 + c;
          if (key >= p.L || (CAUSAL && key > row)) s[c] = -INFINITY;
        }
      }
      // Three-input max tree: a first level of independent maxima over column
      // triples, then levels of three until one value is left.
      float t[(BC + 2) / 3];
#pragma unroll
      for (int i = 0; i < BC / 3; ++i) t[i] = fmax3(s[3 * i], s[3 * i + 1], s[3 * i + 2]);
      int n = BC / 3;
      if (BC % 3 == 1) t[n++] = s[BC - 1];
      if (BC % 3 == 2) t[n++] = fmaxf(s[BC - 2], s[BC - 1]);
#pragma unroll
      for (int level = 0; level < 5; ++level) {
        int m = 0;
#pragma unroll
        for (int i = 0; i + 2 < n; i += 3) t[m++] = fmax3(t[i], t[i + 1], t[i + 2]);
        if (n % 3 == 1) t[m++] = t[n - 1];
        if (n % 3 == 2) t[m++] = fmaxf(t[n - 2], t[n - 1]);
        n = m;
      }
      const float m_loc = t[0] * scale;  // scale > 0
      const bool gvis = j <= my_jmax;
      const bool pass = row_passes_log2(m_loc, m_run, log2_t, t_pos);
      const bool wall = __all_sync(0xffffffffu, !(row_in && gvis) || pass);
      const int fs = vslot(wg, j);
      if (EXT && p.tile_crit) {
        // Largest gap m_local - m_run over the warp's valid rows (log2 units).
        float gap = (!(row_in && gvis) || m_loc == -INFINITY) ? -INFINITY
                    : (m_run == -INFINITY) ? INFINITY : m_loc - m_run;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gap = fmaxf(gap, __shfl_xor_sync(0xffffffffu, gap, o));
        if (lane == 0) wgap[fs + wq] = gap;
      }
      // This warp's loads of S(j) are complete: once all four warps have
      // arrived, the MMA thread may reuse the columns.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        wflag[fs + wq] = wall ? 1 : 0;
        mbar_arrive(b_vote(wg, j));
      }
      // A warp holding a row that did not pass knows at once that its group,
      // and so the tile, is kept.  A warp whose rows all passed reads the
      // other warps' flags.
      bool grp_kept = true, tile_kept = true;
      if (wall) {
        mbar_wait(b_vote(wg, j), vote_par(j), abort_flag);
        int fl[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) fl[q] = wflag[fs + q];
        tile_kept = !(fl[0] & fl[1] & fl[2] & fl[3]);
        grp_kept = false;
#pragma unroll
        for (int q = 0; q < WPG; ++q) grp_kept = grp_kept || fl[grp * WPG + q] == 0;
      }
      // Slice counters: warps holding at least one valid row of a visiting group.
      if (EXT && lane == 0 && gvis && row0 + 128 * wg + wq * 32 < p.L) {
        ++n_svis;
        n_sskip += wall ? 1 : 0;
      }
      if (!tile_kept) {
        warp_signal(b_plo(wg));  // the MMA thread's signal that tile j is skipped
        continue;
      }

      // Block vote: every row of a kept group updates.  Warp vote: only the
      // rows of a warp slice that did not pass.
      const bool mine = row_in && ((EXT && p.slice_vote) ? (gvis && !wall) : grp_kept);
      float alpha = 1.f;
      bool rescale = false;
      if (mine) {
        const float m_new = fmaxf(m_run, m_loc);
        m_run = m_new;
        if (m_ref == -INFINITY) {
          m_ref = m_new;  // first kept tile of the row: its O row is still zero
        } else if (m_new - m_ref > kRescaleLog2) {
          alpha = ex2_approx(m_ref - m_new);
          m_ref = m_new;
          rescale = true;
          l_run *= alpha;
          lr_run *= alpha;
        }
      }
      // P = exp2(S * scale - m_ref) for kept rows, 0 otherwise; bf16 pairs.
      const uint64_t scale2 = f2pack(scale, scale);
      const float nref = mine ? kPackBias - m_ref : -INFINITY;
      const uint64_t nref2 = f2pack(nref, nref);
      __syncwarp();
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds every earlier P.V: S(j) was committed after P.V(j-1).
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o32[32];
          tmem_ld32(tO + c * 32, o32);
          uint32_t w32[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w32[i] = __float_as_uint(o32[i] * alpha);
          tmem_st32(tO + c * 32, w32);
        }
      }
      // No row of this warp takes part (its slice or group skipped the tile,
      // or it is padding): P = 0 without any exponential.
      const bool none = EXT && __all_sync(0xffffffffu, !mine);
      uint64_t sum2v[SSKIP_PF_NACC], sumr2v[SSKIP_PF_NACC];
#pragma unroll
      for (int a = 0; a < SSKIP_PF_NACC; ++a) sum2v[a] = sumr2v[a] = f2pack(0.f, 0.f);
      // P of one half of the keys (HK keys -> HP packed bf16 columns).
      uint32_t pk[HP];
      auto exp_half = [&](int h, const float* sh) {
#pragma unroll
        for (int i = 0; i < HP; ++i) {
          const int c = h * HP + i;  // pair index within the tile
          float p0, p1;
          const uint64_t x2 = ffma2(f2pack(sh[2 * i], sh[2 * i + 1]), scale2, nref2);
          if (exp2_on_fma<D>(c)) {
            f2unpack(exp2_fma2(x2), p0, p1);
          } else {
            float x0, x1;
            f2unpack(x2, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          sum2v[c % SSKIP_PF_NACC] = fadd2(sum2v[c % SSKIP_PF_NACC], f2pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
          if (SSKIP_PF_ROUNDED_L)  // the two bf16 halves widened exactly
            sumr2v[c % SSKIP_PF_NACC] =
                fadd2(sumr2v[c % SSKIP_PF_NACC], f2pack(__uint_as_float(pk[i] << 16),
                                                        __uint_as_float(pk[i] & 0xFFFF0000u)));
        }
      };
      // P of half h lands in columns [h HP, h HP + HP) of the S buffer.
      auto store_half = [&](int h) {
        if constexpr (HP == 32) tmem_st32(tS + h * HP, pk);
        else tmem_st16(tS + h * HP, pk);
      };
      if (none) {
#pragma unroll
        for (int i = 0; i < HP; ++i) pk[i] = 0u;
        store_half(0);
        tmem_st_wait();
        warp_signal(b_plo(wg));
        store_half(1);
        tmem_st_wait();
        warp_signal(b_phi(wg));
      } else if constexpr (kReload<D>() || (EXT && SSKIP_PF_EXT_RELOAD)) {
        // The first half's exponentials use the max pass's registers (already
        // masked); the second half of S is re-read from TMEM (its columns are
        // intact: P of the first half lands in the first quarter), its load in
        // flight while P_lo lands.  Only 64 registers of S stay live past the
        // max pass.
        uint32_t rr[HK];
        exp_half(0, s);
        store_half(0);
        tmem_ld32_async(tS + HK, rr);
        if constexpr (HK == 64) tmem_ld32_async(tS + HK + 32, rr + 32);
        tmem_st_wait();
        warp_signal(b_plo(wg));
        if constexpr (HK == 64) tmem_wait_ld_tie64(rr);
        else tmem_wait_ld_tie32(rr);
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < HK; ++c) {
            const int key = key0 + HK + c;
            if (key >= p.L || (CAUSAL && key > row)) rr[c] = __float_as_uint(-INFINITY);
          }
        }
        exp_half(1, reinterpret_cast<const float*>(rr));
        store_half(1);
        tmem_st_wait();
        warp_signal(b_phi(wg));
      } else {
        // S stays in registers from the max pass (already masked).
        exp_half(0, s);
        store_half(0);
        tmem_st_wait();
        warp_signal(b_plo(wg));
        exp_half(1, s + HK);
        store_half(1);
        tmem_st_wait();
        warp_signal(b_phi(wg));
      }
      if (!none) {
        uint64_t sum2 = sum2v[0], sumr2 = sumr2v[0];
#pragma unroll
        for (int a = 1; a < SSKIP_PF_NACC; ++a) {
          sum2 = fadd2(sum2, sum2v[a]);
          sumr2 = fadd2(sumr2, sumr2v[a]);
        }
        float sa, sb;
        f2unpack(sum2, sa, sb);
        l_run += mine ? (sa + sb) : 0.f;
        f2unpack(sumr2, sa, sb);
        lr_run += mine ? (sa + sb) : 0.f;
      }
    }

    // ---- epilogue: O / l -> bf16, lse = ln 2 * (m_ref + log2 l).
    mbar_wait(b_mmadone, 0, abort_flag);
    tc_fence_after();
    __syncwarp();
    const bool store = row_in && my_jmax >= 0 && n_own > 0 && l_run > 0.f &&
                       dev_check(row < p.L && hq < p.Hq);
    if (n_own > 0) {
      const float inv_l = store ? 1.f / (SSKIP_PF_ROUNDED_L ? lr_run : l_run) : 0.f;
      __nv_bfloat16* orow = p.o + (((size_t)b * p.Hq + hq) * p.L + (store ? row : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o32[32];
        tmem_ld32(tO + c * 32, o32);
        if (store) {
          uint4 w4[4];
          uint32_t* wp = reinterpret_cast<uint32_t*>(w4);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            wp[i] = pack_bf16x2(o32[2 * i] * inv_l, o32[2 * i + 1] * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = w4[i];
        }
      }
    }
    if (store)
      p.lse[((size_t)b * p.Hq + hq) * p.L + row] =
          (m_ref - kPackBias + __log2f(l_run)) * 0.69314718055994531f;
    if (EXT && lane == 0 && p.counts && p.n_counts == 4 && p.slice_vote && n_svis > 0) {
      atomicAdd(&p.counts[2], (unsigned long long)n_sskip);
      atomicAdd(&p.counts[3], (unsigned long long)n_svis);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace sskip
