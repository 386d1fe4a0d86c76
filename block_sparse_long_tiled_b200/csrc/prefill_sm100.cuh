// prefill_sm100.cuh -- Skip-Softmax tiled attention prefill for sm_100a.
//
// The FlashAttention carrier of the TensorRT-LLM Skip-Softmax article
// ("Skip Softmax 到底怎么回事" section: logits, then softmax, then x V), with
// the block test of its "Skip Softmax 的三步走算法" section inserted between
// the two contractions: a key tile whose rows all sit more than ln(1/t) below
// their running maximum skips its softmax, its P.V (BMM2) and its V load.
//
// One CTA owns 128 query rows of one (batch, query head): a single 128-row
// tile when Br = 128, or two stacked 64-row tiles (each voting on its own)
// when Br = 64.  Warp roles (256 threads):
//   warp 0      TMA producer: Q once, then K tiles through an NK-stage ring.
//   warp 1      TMEM allocator and the single thread that issues tcgen05.mma:
//               S_{j+1} = Q K_{j+1}^T is issued before P_j is ready, so the
//               tensor core computes the next logits while softmax runs.
//   warps 4..7  softmax warpgroup, thread r owns TMEM lane (row) r: loads its S
//               row, masks it, takes its local max, votes; the warpgroup's
//               vote decides the tile; for a kept tile thread 0 of the group
//               issues the V TMA at once, the rows compute P = exp2(S - m) in
//               fp32, pack it to bf16 in place of S in TMEM, and the MMA
//               thread runs O += P V_j with P read from TMEM.
// Skipped tiles therefore cost one QK^T MMA and one row max: no exp, no P
// store, no V bytes, no P.V.
//
// Exponent reference: the vote always uses the exact running max m_run; the
// exponentials use a reference m_ref that is raised only when m_run exceeds
// it by more than 8 (log2 units), so O in TMEM is rescaled rarely.  The final
// O / l and lse = ln 2 * (m_ref + log2 l) are independent of that choice.
#pragma once

#include "sm100_ptx.cuh"
#include "skip_rule.cuh"

namespace sskip {

struct PrefillParams {
  __nv_bfloat16* o;            // [B, Hq, L, D]
  float* lse;                  // [B, Hq, L]
  unsigned long long* counts;  // {skipped, visited} or null
  uint8_t* tile_state;         // [B, Hq, n_q, n_k] or null
  int B, Hq, Hkv, L, G;
  int n_q;                     // ceil(L / Br)
  int n_k;                     // ceil(L / Bc)
  int n_units;                 // ceil(L / 128): 128-row units per head
  float scale_log2;            // sm_scale * log2(e)
  float log2_t;                // log2(tsf / L), -inf when tsf == 0
  int t_positive;
};

constexpr int kPfThreads = 256;
constexpr float kRescaleLog2 = 8.0f;

template <int D, int BC>
struct PrefillCfg {
  static constexpr int kNK = (D * BC >= 128 * 128) ? 3 : 4;  // K stages
  static constexpr int kNV = (D * BC >= 128 * 128) ? 2 : 3;  // V stages
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = BC * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kNK * kKVBytes;
  static constexpr int kBar = kV + kNV * kKVBytes;
  // barriers: q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  //           s_full[2], dec_full[2], o_done, mma_done
  static constexpr int kNumBars = 1 + 2 * kNK + 2 * kNV + 2 + 2 + 1 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // dec_kept[2], vote[4], tmem, abort
  static constexpr int kTotal = kMisc + 64;
  static constexpr int kAlloc = kTotal + 1024;  // room to align the base to 1 KB
  static constexpr int kTmemCols = (2 * BC + D) <= 256 ? 256 : 512;
  static_assert(kQBytes % 1024 == 0 && kKVBytes % 1024 == 0, "tiles must keep 1 KB alignment");
  static_assert(kTotal <= 227 * 1024, "shared memory budget");
};

template <int D, int BR, int BC, bool CAUSAL>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D, BC>;
  constexpr int NK = C::kNK, NV = C::kNV;
  constexpr int NGRP = 128 / BR;  // vote groups per CTA
  constexpr int WPG = BR / 32;    // warps per vote group
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BC, 0, 0);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 0, 1);
  static_assert(BR == 64 || BR == 128, "Br");
  static_assert(BC == 64 || BC == 128, "Bc");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  int* misc = reinterpret_cast<int*>(smem + C::kMisc);
  int* dec_kept = misc;           // [2]
  // Vote flags, double-buffered by tile parity: after a skipped tile there is
  // no second barrier, so a fast warp may post tile j+1's flag while a slow
  // warp still reads tile j's.
  int* vote_s = misc + 2;         // [2][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 10);
  volatile int* abort_flag = misc + 11;

  const uint32_t b_qfull = smem_u32(&bars[0]);
  auto b_kfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_kempty = [&](int s) { return smem_u32(&bars[1 + NK + s]); };
  auto b_vfull = [&](int s) { return smem_u32(&bars[1 + 2 * NK + s]); };
  auto b_vempty = [&](int s) { return smem_u32(&bars[1 + 2 * NK + NV + s]); };
  auto b_sfull = [&](int s) { return smem_u32(&bars[1 + 2 * NK + 2 * NV + s]); };
  auto b_dec = [&](int s) { return smem_u32(&bars[1 + 2 * NK + 2 * NV + 2 + s]); };
  const uint32_t b_odone = smem_u32(&bars[1 + 2 * NK + 2 * NV + 4]);
  const uint32_t b_mmadone = smem_u32(&bars[1 + 2 * NK + 2 * NV + 5]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: heaviest causal rows first across all heads.
  const int bh_count = p.B * p.Hq;
  const int ublk = blockIdx.x / bh_count;
  const int i128 = CAUSAL ? (p.n_units - 1 - ublk) : ublk;
  const int bh = blockIdx.x % bh_count;
  const int b = bh / p.Hq, hq = bh % p.Hq, kvh = hq / p.G;
  const int row0 = i128 * 128;
  const int n_j = CAUSAL ? min(p.n_k, (row0 + 127) / BC + 1) : p.n_k;

  if (threadIdx.x == 0) {
    mbar_init(b_qfull, 1);
    for (int s = 0; s < NK; ++s) { mbar_init(b_kfull(s), 1); mbar_init(b_kempty(s), 1); }
    for (int s = 0; s < NV; ++s) { mbar_init(b_vfull(s), 1); mbar_init(b_vempty(s), 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(b_sfull(s), 1); mbar_init(b_dec(s), 1); }
    mbar_init(b_odone, 1);
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
  const uint32_t tmem_o = tmem + 2 * BC;

  if (warp == 0) {
    // ================= TMA producer: Q once, then the K ring =================
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(b_qfull, C::kQBytes);
#pragma unroll
      for (int blk = 0; blk < D / 64; ++blk)
        tma_load_3d(sbase + C::kQ + blk * 128 * 128, &tmQ, b_qfull, blk * 64, row0, b * p.Hq + hq);
      int last = -1;
      for (int j = 0; j < n_j; ++j) {
        const int s = j % NK;
        if (j >= NK && !mbar_wait(b_kempty(s), ((j / NK) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(b_kfull(s), C::kKVBytes);
#pragma unroll
        for (int blk = 0; blk < D / 64; ++blk)
          tma_load_3d(sbase + C::kK + s * C::kKVBytes + blk * BC * 128, &tmK, b_kfull(s), blk * 64,
                      j * BC, b * p.Hkv + kvh);
        last = j;
      }
      // Never leave with copies in flight: wait (bounded, even when aborting)
      // for the last ring's worth of K copies.
      if (*abort_flag) {
        int dummy = 0;
        for (int j = max(0, last - NK + 1); j <= last; ++j)
          mbar_wait(b_kfull(j % NK), (j / NK) & 1, &dummy);
        mbar_wait(b_qfull, 0, &dummy);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      auto issue_s = [&](int j) {
        const int s = j % NK;
        const uint32_t d_tmem = tmem + (j & 1) * BC;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a = sbase + C::kQ + (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          const uint32_t bk = sbase + C::kK + s * C::kKVBytes + (kk >> 2) * (BC * 128) + (kk & 3) * 32;
          umma_ss(d_tmem, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(bk, 16, 1024), IDESC_S,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(b_sfull(j & 1));
        umma_commit(b_kempty(s));
      };
      bool ok = mbar_wait(b_qfull, 0, abort_flag);
      ok = ok && mbar_wait(b_kfull(0), 0, abort_flag);
      tc_fence_after();
      if (ok) issue_s(0);
      int kc = 0;
      for (int j = 0; ok && j < n_j; ++j) {
        if (j + 1 < n_j) {
          if (!mbar_wait(b_kfull((j + 1) % NK), ((j + 1) / NK) & 1, abort_flag)) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!mbar_wait(b_dec(j & 1), (j >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        if (dec_kept[j & 1]) {
          const int vs = kc % NV;
          if (!mbar_wait(b_vfull(vs), (kc / NV) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t p_tmem = tmem + (j & 1) * BC;
#pragma unroll
          for (int kk = 0; kk < BC / 16; ++kk) {
            const uint32_t bv = sbase + C::kV + vs * C::kKVBytes + kk * 16 * 128;
            umma_ts(tmem_o, p_tmem + kk * 8, smem_desc_sw128(bv, BC * 128, 1024), IDESC_PV,
                    (kc > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(b_vempty(vs));
          umma_commit(b_odone);
          ++kc;
        }
      }
      // Drain: every MMA issued by this thread completes before TMEM is freed.
      umma_commit(b_mmadone);
      int dummy = 0;
      mbar_wait(b_mmadone, 0, &dummy);
    }
  } else if (warp >= 4) {
    // ================= softmax warpgroup =================
    const int r = (warp - 4) * 32 + lane;  // TMEM lane == row within the unit
    const int grp = r / BR;
    const int row = row0 + r;
    const bool row_in = row < p.L;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    // Per group: does the query tile exist, and its last visited key tile.
    int g_tile[NGRP], g_jmax[NGRP];
#pragma unroll
    for (int g = 0; g < NGRP; ++g) {
      g_tile[g] = i128 * NGRP + g;
      const bool exists = g_tile[g] < p.n_q;
      const int jm = CAUSAL ? min(p.n_k - 1, ((g_tile[g] + 1) * BR - 1) / BC) : p.n_k - 1;
      g_jmax[g] = exists ? jm : -1;
    }
    const bool elected = (warp == 4 && lane == 0);
    const float log2_t = p.log2_t;
    const bool t_pos = p.t_positive != 0;

    float m_run = -INFINITY, m_ref = -INFINITY, l_run = 0.f;
    int kc = 0;                 // PVs issued so far (kept tiles)
    uint32_t o_phase = 0;
    long long n_vis = 0, n_skip = 0;
    int last_v = -1;

    for (int j = 0; j < n_j; ++j) {
      const int sb = j & 1;
      mbar_wait(b_sfull(sb), (j >> 1) & 1, abort_flag);
      tc_fence_after();
      __syncwarp();  // tcgen05.ld is warp-collective; lane 0 ran alone above
      float s[BC];
#pragma unroll
      for (int c = 0; c < BC / 32; ++c) {
        float t32[32];
        tmem_ld32(tmem + lane_base + sb * BC + c * 32, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = t32[i];
      }
      // Mask: keys past L, and keys after the row in causal attention.
      const int key0 = j * BC;
      const bool need_mask = (key0 + BC > p.L) || (CAUSAL && key0 + BC - 1 > row);
      float mx = -INFINITY;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BC; ++c) {
          const int key = key0 + c;
          if (key >= p.L || (CAUSAL && key > row)) s[c] = -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BC; ++c) mx = fmaxf(mx, s[c]);
      }
      const float m_loc = mx * p.scale_log2;  // scale > 0 keeps the argmax
      const bool gvis = j <= g_jmax[grp];
      const bool pass = row_passes_log2(m_loc, m_run, log2_t, t_pos);
      const bool ok = !(row_in && gvis) || pass;
      const bool wall = __all_sync(0xffffffffu, ok);
      if (lane == 0) vote_s[sb * 4 + warp - 4] = wall ? 1 : 0;
      tc_fence_before();
      named_bar_sync(1, 128);
      bool g_kept[NGRP];
      bool tile_kept = false;
#pragma unroll
      for (int g = 0; g < NGRP; ++g) {
        bool all = true;
#pragma unroll
        for (int w = 0; w < WPG; ++w) all = all && (vote_s[sb * 4 + g * WPG + w] != 0);
        const bool vis = j <= g_jmax[g];
        g_kept[g] = vis && !all;
        tile_kept = tile_kept || g_kept[g];
        if (elected && vis) {
          ++n_vis;
          n_skip += all ? 1 : 0;
          if (p.tile_state)
            p.tile_state[(((size_t)b * p.Hq + hq) * p.n_q + g_tile[g]) * p.n_k + j] = all ? 2 : 1;
        }
      }
      if (elected && tile_kept && !*abort_flag) {
        // The vote is in: request V_j now, ahead of the exponentials.
        const int vs = kc % NV;
        if (kc < NV || mbar_wait(b_vempty(vs), ((kc / NV) - 1) & 1, abort_flag)) {
          mbar_arrive_expect_tx(b_vfull(vs), C::kKVBytes);
#pragma unroll
          for (int blk = 0; blk < D / 64; ++blk)
            tma_load_3d(sbase + C::kV + vs * C::kKVBytes + blk * BC * 128, &tmV, b_vfull(vs),
                        blk * 64, key0, b * p.Hkv + kvh);
          last_v = kc;
        }
      }

      if (tile_kept) {
        const bool mine = g_kept[grp] && row_in;
        float alpha = 1.f;
        bool rescale = false;
        if (mine) {
          const float m_new = fmaxf(m_run, m_loc);
          m_run = m_new;
          if (m_ref == -INFINITY) {
            m_ref = m_new;  // first kept tile of the row: O row is still zero
          } else if (m_new - m_ref > kRescaleLog2) {
            alpha = ex2_approx(m_ref - m_new);
            m_ref = m_new;
            rescale = true;
            l_run *= alpha;
          }
        }
        // P = exp2(S * scale - m_ref), packed two bf16 per TMEM column.
        const float neg_ref = mine ? -m_ref : 0.f;
        float rowsum = 0.f;
        uint32_t pk[BC / 2];
#pragma unroll
        for (int c = 0; c < BC / 2; ++c) {
          float p0 = 0.f, p1 = 0.f;
          if (mine) {
            p0 = ex2_approx(fmaf(s[2 * c], p.scale_log2, neg_ref));
            p1 = ex2_approx(fmaf(s[2 * c + 1], p.scale_log2, neg_ref));
          }
          rowsum += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_run += rowsum;
        // The previous P.V must be complete before O is touched (and this
        // keeps the o_done phase count exact: one wait per issued P.V).
        if (kc > 0) {
          mbar_wait(b_odone, o_phase, abort_flag);
          o_phase ^= 1u;
          tc_fence_after();
        }
        __syncwarp();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o32[32];
            tmem_ld32(tmem_o + lane_base + c * 32, o32);
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o32[i] * alpha);
            tmem_st32(tmem_o + lane_base + c * 32, w);
          }
        }
#pragma unroll
        for (int c = 0; c < BC / 64; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = pk[c * 32 + i];
          tmem_st32(tmem + lane_base + sb * BC + c * 32, w);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar_sync(1, 128);
        ++kc;
      }
      if (elected) {
        dec_kept[sb] = tile_kept ? 1 : 0;
        mbar_arrive(b_dec(sb));
      }
    }

    // ---- epilogue: O / l -> bf16, lse = ln 2 * (m_ref + log2 l).
    if (kc > 0) {
      mbar_wait(b_odone, o_phase, abort_flag);
      tc_fence_after();
    }
    __syncwarp();
    const bool store = row_in && g_jmax[grp] >= 0 && kc > 0;
    const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
    __nv_bfloat16* orow = p.o + (((size_t)b * p.Hq + hq) * p.L + (store ? row : 0)) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o32[32];
      tmem_ld32(tmem_o + lane_base + c * 32, o32);
      if (store) {
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int i = 0; i < 16; ++i) wp[i] = pack_bf16x2(o32[2 * i] * inv_l, o32[2 * i + 1] * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = w[i];
      }
    }
    if (store)
      p.lse[((size_t)b * p.Hq + hq) * p.L + row] = (m_ref + __log2f(l_run)) * 0.69314718055994531f;
    if (elected) {
      if (p.counts) {
        atomicAdd(&p.counts[0], (unsigned long long)n_skip);
        atomicAdd(&p.counts[1], (unsigned long long)n_vis);
      }
      if (*abort_flag) {  // leave no V copy in flight
        int dummy = 0;
        for (int k = max(0, last_v - NV + 1); k <= last_v; ++k)
          mbar_wait(b_vfull(k % NV), (k / NV) & 1, &dummy);
      }
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
