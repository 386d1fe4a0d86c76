// decode_sm100.cuh -- split-KV Skip-Softmax decode for sm_100a.
//
// One CTA per (split, kv head, batch).  Its G = Hq / Hkv query heads share the
// kv head, so every key tile (Bc = 64 keys) gets ONE joint decision and a
// skipped tile costs no V bytes at all -- the bandwidth saving the
// TensorRT-LLM Skip-Softmax article claims for decode ("Skip Softmax 带来了
// 哪些实战好处" section: decode is bound by reading the KV cache; skipping
// avoids loading the V blocks).
//
// Decode is HBM-bound (about 4 FLOP per cache byte), so the two contractions
// run on CUDA cores and the design keeps HBM busy and the per-tile critical
// path short:
//   * K tiles stream through a ring of 1-D bulk-async copies issued NK tiles
//     ahead;
//   * each of the 8 warps scores 8 of the tile's 64 keys (8 lanes per key, a
//     transpose-reduce leaves one head's dot product per lane) and publishes
//     its per-head maxima; after ONE block barrier every warp reads the eight
//     maxima and takes the same joint decision itself -- no warp waits on a
//     voting warp;
//   * the V copy of a kept tile is issued right after that barrier, LAG tiles
//     before its P.V runs (a decision needs only the K side);
//   * each warp keeps P, its partial row sums and its partial O for its own
//     keys, so P never crosses warps; the partials merge once per split.
// The split's normalised partial O_s and lse_s (fp32) go to the workspace; a
// second kernel merges the splits by log-sum-exp.
#pragma once

#include "sm100_ptx.cuh"
#include "skip_rule.cuh"

namespace sskip {

struct DecodeParams {
  const __nv_bfloat16* q;    // [B, Hq, D]
  const __nv_bfloat16* kc;   // [B, Hkv, Lmax, D]
  const __nv_bfloat16* vc;   // [B, Hkv, Lmax, D]
  const int* seqlens;        // [B]
  float* o_part;             // [B, Hq, S, D]
  float* lse_part;           // [B, Hq, S], natural log
  __nv_bfloat16* o;          // [B, Hq, D]
  float* lse;                // [B, Hq]
  unsigned long long* counts;  // {skipped, visited} or null
  uint8_t* tile_state;       // [B, Hkv, n_k_max] or null
  float* tile_crit;          // [B, Hkv, n_k_max] or null: ln of the skipping factor
  int B, Hq, Hkv, Lmax, S, n_k_max;
  float scale_log2;          // sm_scale * log2(e)
  float tsf;                 // threshold_scale_factor
};

constexpr int kDecBc = 64;
constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecNK = 3;    // K ring stages
constexpr int kDecLag = 2;   // P.V runs this many tiles behind the decision
constexpr int kDecNV = 3;    // V ring stages (> kDecLag)
constexpr int kDecNPB = kDecLag + 1;  // per-warp P ring
constexpr int kDecKeysPerWarp = kDecBc / kDecWarps;  // 8

template <int D, int G>
struct DecodeSmem {
  static constexpr int kTileBytes = kDecBc * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kDecNK * kTileBytes;
  static constexpr int kP = kV + kDecNV * kTileBytes;                        // [W][NPB][8][G]
  static constexpr int kAlpha = kP + kDecWarps * kDecNPB * kDecKeysPerWarp * G * 4;  // [W][NPB][G]
  static constexpr int kWmax = kAlpha + kDecWarps * kDecNPB * G * 4;        // [2][G][W]
  static constexpr int kLsum = kWmax + 2 * G * kDecWarps * 4;               // [W][G]
  static constexpr int kBar = (kLsum + kDecWarps * G * 4 + 15) / 16 * 16;
  static constexpr int kTotal = kBar + (kDecNK + kDecNV) * 8 + 16;
  // The cross-warp reduction of O at the end reuses the K ring.
  static_assert(kDecWarps * G * D * 4 <= kDecNK * kTileBytes, "reduction scratch fits the K ring");
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// Reduce G partial dot products over the 8 lanes of a key group so that lane
// `sub` ends with the full sum for head sub / (8 / G): at each halving step a
// lane keeps the half of the heads selected by its lane bit and receives the
// partner's partials of that half; once one head is left the remaining lane
// bits all-reduce it.
template <int G>
__device__ __forceinline__ float transpose_reduce8(const float (&acc)[G], int sub) {
  float v[G];
#pragma unroll
  for (int g = 0; g < G; ++g) v[g] = acc[g];
  int width = G;
#pragma unroll
  for (int m = 4; m >= 1; m >>= 1) {
    if (width > 1) {
      const int half = width / 2;
      const bool upper = (sub & m) != 0;
#pragma unroll
      for (int i = 0; i < (G > 1 ? G / 2 : 1); ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      width = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
  return v[0];
}

// CRIT = true adds the critical-value record; the plain kernel is built
// without it (the extra branch in the tile loop costs time even when off).
// Eight heads at d = 128 keep 128 registers of q and 32 of accumulators per
// thread, more than two CTAs per SM leave (128); they run one CTA per SM.
template <int D, int G>
constexpr int dec_ctas_per_sm() { return (G * D > 512) ? 1 : 2; }

template <int D, int G, bool CRIT>
__global__ void __launch_bounds__(kDecThreads, dec_ctas_per_sm<D, G>())
    decode_split_kernel(const DecodeParams p) {
  using L = DecodeSmem<D, G>;
  constexpr int PPL = D / 64;        // 16-byte pieces per lane per key (8 lanes per key)
  constexpr int EPL = D / 32;        // P.V output elements per lane
  constexpr int LPH = 8 / G;         // lanes per head after the transpose-reduce
  extern __shared__ __align__(1024) uint8_t smem[];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // seqlens[b] must lie in [1, Lmax]. A length outside that range is latched
  // as an invalid argument and clamped to it, so no copy leaves the sequence's
  // [Lmax, d] slab and no record index leaves [0, ceil(Lmax / Bc)); a length
  // of 0 leaves every split empty.
  const int Lraw = p.seqlens[b];
  if ((Lraw < 1 || Lraw > p.Lmax) && tid == 0 && split == 0 && kvh == 0)
    latch_status(kStatusInvalidArg);
  const int Lb = min(max(Lraw, 0), p.Lmax);
  const int n_k = (Lb + kDecBc - 1) / kDecBc;
  const int c_per = (n_k + p.S - 1) / p.S;
  const int j0 = split * c_per;
  const int ntiles = max(0, min(n_k, j0 + c_per) - j0);
  const size_t head0 = (size_t)b * p.Hq + (size_t)kvh * G;
  if (!dev_check(b < p.B && kvh < p.Hkv && split < p.S && head0 + G <= (size_t)p.B * p.Hq &&
                 kvh * G + G <= p.Hq))
    return;  // the whole CTA, before any barrier

  if (ntiles == 0) {  // an empty split contributes nothing to the merge
    for (int i = tid; i < G * D; i += kDecThreads)
      p.o_part[((head0 + i / D) * p.S + split) * D + (i % D)] = 0.f;
    if (tid < G) p.lse_part[(head0 + tid) * p.S + split] = -INFINITY;
    return;
  }

  float* Pbuf = reinterpret_cast<float*>(smem + L::kP) + warp * kDecNPB * kDecKeysPerWarp * G;
  float* Abuf = reinterpret_cast<float*>(smem + L::kAlpha) + warp * kDecNPB * G;
  float* wmax = reinterpret_cast<float*>(smem + L::kWmax);
  float* lsum = reinterpret_cast<float*>(smem + L::kLsum);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + L::kBar + (kDecNK + kDecNV) * 8);
  const uint32_t k_smem = smem_u32(smem + L::kK);
  const uint32_t v_smem = smem_u32(smem + L::kV);
  auto kfull = [&](int s) { return smem_u32(&bars[s]); };
  auto vfull = [&](int s) { return smem_u32(&bars[kDecNK + s]); };

  const size_t cache_head = ((size_t)b * p.Hkv + kvh) * (size_t)p.Lmax;
  const __nv_bfloat16* kbase = p.kc + cache_head * D;
  const __nv_bfloat16* vbase = p.vc + cache_head * D;
  auto tile_keys = [&](int t) { return min(kDecBc, Lb - (j0 + t) * kDecBc); };

  if (tid == 0) {
    for (int s = 0; s < kDecNK + kDecNV; ++s) mbar_init(smem_u32(&bars[s]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](uint32_t ring, int stage, uint32_t bar, const __nv_bfloat16* base, int t) {
    const uint32_t bytes = (uint32_t)tile_keys(t) * D * 2;
    if (!dev_check(j0 + t < n_k && (j0 + t) * kDecBc + tile_keys(t) <= p.Lmax && bytes > 0)) {
      mbar_arrive(bar);  // the phase completes without data
      return;
    }
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(ring + stage * L::kTileBytes, base + (size_t)(j0 + t) * kDecBc * D, bytes, bar);
  };
  // Thread 0 issues every copy and keeps what an aborting CTA needs to wait
  // them out before it exits: the number of K tiles issued (tiles go out in
  // order) and, per V slot, whether it was used and the parity of its copies.
  int k_issued = 0;
  uint32_t v_used = 0, v_par = 0;
  auto issue_k = [&](int t) {
    issue(k_smem, t % kDecNK, kfull(t % kDecNK), kbase, t);
    k_issued = t + 1;
  };
  auto issue_v = [&](int t) {
    issue(v_smem, t % kDecNV, vfull(t % kDecNV), vbase, t);
    v_used |= 1u << (t % kDecNV);
    v_par ^= 1u << (t % kDecNV);
  };
  if (tid == 0)
    for (int t = 0; t < min(kDecNK, ntiles); ++t) issue_k(t);

  // Lane layout of the scores: 8 lanes per key (sub = lane % 8), 4 keys per
  // warp per pass; pass ps covers keys ps*32 + warp*4 + lane/8.
  const int sub = lane & 7, kq = lane >> 3;
  const int hs = sub / LPH;             // head whose score this lane holds
  const bool owner = (sub % LPH) == 0;  // one writer per (key, head)
  const int hv = lane % G;              // head this lane votes / keeps state for
  // q as fp32 pairs: the dot products run as packed f32x2 FMAs.
  uint64_t qreg[G][PPL * 4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
      const uint4 w = *reinterpret_cast<const uint4*>(p.q + (head0 + g) * D + (sub + 8 * i) * 8);
      float f[8];
      bf16x8_to_f32(w, f);
#pragma unroll
      for (int e = 0; e < 4; ++e) qreg[g][i * 4 + e] = f2pack(f[2 * e], f[2 * e + 1]);
    }

  const bool t_positive = p.tsf > 0.f;
  const float log2_t = t_positive ? (float)log2((double)p.tsf / (double)Lb) : -INFINITY;
  float m_run = -INFINITY;  // running max of head hv (identical in every warp)
  float l_lane = 0.f;       // this lane's share of the row sum of head hs
  uint64_t oacc[G][EPL / 2];  // fp32 pairs of this lane's output columns
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) oacc[g][e] = f2pack(0.f, 0.f);
  uint32_t v_phase = 0;      // one parity bit per V slot
  uint64_t kept_mask = 0;    // bit (t % 64): tile t was kept
  int n_skipped = 0;

  // A bounded wait that runs out raises the CTA's abort flag; from then on
  // every wait returns at once, no new copy is issued and the loop runs out
  // its remaining tiles on meaningless data (the outputs are undefined, the
  // status word says why).  Copies already in flight are waited out after
  // the loop.
  for (int t = 0; t < ntiles + kDecLag; ++t) {
    float s[2] = {-INFINITY, -INFINITY};
    const bool live = t < ntiles;
    if (live) {
      // ---- scores of this warp's 8 keys, in log2 units; keys past L_b -> -inf.
      const int ks = t % kDecNK;
      mbar_wait(kfull(ks), (t / kDecNK) & 1, abort_flag);
      const int keys = tile_keys(t);
      const uint8_t* ktile = smem + L::kK + ks * L::kTileBytes;
      float mx = -INFINITY;
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        const int key = ps * 32 + warp * 4 + kq;
        uint64_t acc2[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc2[g] = f2pack(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
          const uint4 w =
              *reinterpret_cast<const uint4*>(ktile + key * D * 2 + (sub + 8 * i) * 16);
          float f[8];
          bf16x8_to_f32(w, f);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t k2 = f2pack(f[2 * e], f[2 * e + 1]);
#pragma unroll
            for (int g = 0; g < G; ++g) acc2[g] = ffma2(qreg[g][i * 4 + e], k2, acc2[g]);
          }
        }
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float lo, hi;
          f2unpack(acc2[g], lo, hi);
          acc[g] = lo + hi;
        }
        const float dot = transpose_reduce8<G>(acc, sub);
        s[ps] = (key < keys) ? dot * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[ps]);
      }
      // per-head max over the warp's 4 key groups (lane bits 3, 4)
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (kq == 0 && owner) wmax[((t & 1) * G + hs) * kDecWarps + warp] = mx;
    }
    __syncthreads();  // maxima of tile t published; K slot t % NK free; P.V of t-1-LAG done

    if (live) {
      if (tid == 0 && t + kDecNK < ntiles && !*abort_flag) issue_k(t + kDecNK);
      // ---- the joint decision, taken identically by every warp.
      const float* wm = wmax + ((t & 1) * G + hv) * kDecWarps;
      float m_loc = wm[0];
#pragma unroll
      for (int w = 1; w < kDecWarps; ++w) m_loc = fmaxf(m_loc, wm[w]);
      const bool skip =
          __all_sync(0xffffffffu, row_passes_log2(m_loc, m_run, log2_t, t_positive));
      if (CRIT && warp == 0) {
        // Critical factor: the tile is skipped iff ln(tsf) > max over the G
        // heads of (m_local - m_run) + ln(L_b) (any factor while t_b < 1).
        float gap = (m_loc == -INFINITY) ? -INFINITY
                    : (m_run == -INFINITY) ? INFINITY : m_loc - m_run;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gap = fmaxf(gap, __shfl_xor_sync(0xffffffffu, gap, o));
        if (lane == 0 && dev_check(j0 + t < p.n_k_max))
          p.tile_crit[((size_t)b * p.Hkv + kvh) * p.n_k_max + j0 + t] =
              gap * 0.69314718055994531f + logf((float)Lb);
      }
      if (!skip) {
        const float m_new = fmaxf(m_run, m_loc);
        const float a = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
        m_run = m_new;
        const float mh = __shfl_sync(0xffffffffu, m_new, hs);  // lane hs holds head hs
        const float ah = __shfl_sync(0xffffffffu, a, hs);
        const float p0 = ex2_approx(s[0] - mh), p1 = ex2_approx(s[1] - mh);
        l_lane = ah * l_lane + p0 + p1;
        float* Pt = Pbuf + (t % kDecNPB) * kDecKeysPerWarp * G;
        if (owner) {
          Pt[kq * G + hs] = p0;
          Pt[(4 + kq) * G + hs] = p1;
        }
        if (lane < G) Abuf[(t % kDecNPB) * G + lane] = a;
        kept_mask |= 1ull << (t & 63);
        if (tid == 0 && !*abort_flag) issue_v(t);
      } else {
        kept_mask &= ~(1ull << (t & 63));
        n_skipped += 1;
      }
      if (tid == 0 && p.tile_state && dev_check(j0 + t < p.n_k_max))
        p.tile_state[((size_t)b * p.Hkv + kvh) * p.n_k_max + j0 + t] = skip ? 2 : 1;
    }

    const int u = t - kDecLag;
    if (u >= 0 && ((kept_mask >> (u & 63)) & 1)) {
      // ---- O = alpha O + P_u V_u over this warp's 8 keys.
      const int vs = u % kDecNV;
      mbar_wait(vfull(vs), (v_phase >> vs) & 1, abort_flag);
      v_phase ^= 1u << vs;
      __syncwarp();
      const int keys = tile_keys(u);
      const float* Pu = Pbuf + (u % kDecNPB) * kDecKeysPerWarp * G;
      const uint8_t* vtile = smem + L::kV + vs * L::kTileBytes;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float a = Abuf[(u % kDecNPB) * G + g];
        const uint64_t a2 = f2pack(a, a);
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e) oacc[g][e] = fmul2(oacc[g][e], a2);
      }
#pragma unroll
      for (int k = 0; k < kDecKeysPerWarp; ++k) {
        const int key = (k >> 2) * 32 + warp * 4 + (k & 3);
        if (key < keys) {
          float vf[EPL];
          if constexpr (EPL == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(vtile + key * D * 2 + lane * 8);
            vf[0] = __uint_as_float(w.x << 16);
            vf[1] = __uint_as_float(w.x & 0xFFFF0000u);
            vf[2] = __uint_as_float(w.y << 16);
            vf[3] = __uint_as_float(w.y & 0xFFFF0000u);
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(vtile + key * D * 2 + lane * 4);
            vf[0] = __uint_as_float(w << 16);
            vf[1] = __uint_as_float(w & 0xFFFF0000u);
          }
          uint64_t v2[EPL / 2];
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e) v2[e] = f2pack(vf[2 * e], vf[2 * e + 1]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pk = Pu[k * G + g];
            const uint64_t p2 = f2pack(pk, pk);
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) oacc[g][e] = ffma2(p2, v2[e], oacc[g][e]);
          }
        }
      }
    }
  }

  // ---- epilogue: merge the warps' partial O and row sums, write the split.
  // A lane's row-sum share counts once per (key group, head).
  float lw = owner ? l_lane : 0.f;
  lw += __shfl_xor_sync(0xffffffffu, lw, 8);
  lw += __shfl_xor_sync(0xffffffffu, lw, 16);
  __syncthreads();  // every warp is past its last use of the K ring (and its last wait)
  if (*abort_flag) {
    // Every wait is over, so the flag is final here.  Wait out each ring
    // slot's last copy (those a timed-out wait did not see land) before the
    // CTA exits and its shared memory is reused.
    if (tid == 0) {
      int no_abort = 0;
#pragma unroll
      for (int s = 0; s < kDecNK; ++s)
        if (k_issued > s) {  // the last K tile that went to slot s
          const int t_last = s + (k_issued - 1 - s) / kDecNK * kDecNK;
          mbar_wait(kfull(s), (t_last / kDecNK) & 1, &no_abort);
        }
#pragma unroll
      for (int s = 0; s < kDecNV; ++s)  // the phase of the slot's last copy
        if ((v_used >> s) & 1) mbar_wait(vfull(s), ((v_par >> s) & 1) ^ 1, &no_abort);
    }
    return;
  }
  float* red = reinterpret_cast<float*>(smem + L::kK);
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) {
      float lo, hi;
      f2unpack(oacc[g][e], lo, hi);
      red[(warp * G + g) * D + lane * EPL + 2 * e] = lo;
      red[(warp * G + g) * D + lane * EPL + 2 * e + 1] = hi;
    }
  if (kq == 0 && owner) lsum[warp * G + hs] = lw;
  if (tid == 0 && p.counts) {
    atomicAdd(&p.counts[0], (unsigned long long)n_skipped);
    atomicAdd(&p.counts[1], (unsigned long long)ntiles);
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, e = i % D;
    float acc = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      acc += red[(w * G + g) * D + e];
      l += lsum[w * G + g];
    }
    p.o_part[((head0 + g) * p.S + split) * D + e] = acc / l;
  }
  if (tid < G) {
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) l += lsum[w * G + tid];
    // lanes tid < G of warp 0 hold the running max of head tid
    p.lse_part[(head0 + tid) * p.S + split] = (m_run + __log2f(l)) * 0.69314718055994531f;
  }
}

// Merge the splits of one (batch, query head): lse = log sum_s exp(lse_s),
// O = sum_s exp(lse_s - lse) O_s.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const size_t bh = blockIdx.x;
  if (!dev_check(bh < (size_t)p.B * p.Hq)) return;
  const float* lp = p.lse_part + bh * p.S;
  __shared__ float w_s[64];
  __shared__ float lse_s;
  if (threadIdx.x < 32) {
    float mx = -INFINITY;
    for (int s = threadIdx.x; s < p.S; s += 32) mx = fmaxf(mx, lp[s]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float sum = 0.f;
    for (int s = threadIdx.x; s < p.S; s += 32) {
      const float e = (lp[s] == -INFINITY) ? 0.f : __expf(lp[s] - mx);
      w_s[s] = e;
      sum += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    // Every split empty (a sequence of length 0, or aborted splits): O = 0
    // and lse = -inf rather than 0 / 0.
    if (threadIdx.x == 0) lse_s = sum > 0.f ? mx + __logf(sum) : -INFINITY;
    __syncwarp();
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int s = threadIdx.x; s < p.S; s += 32) w_s[s] *= inv;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < p.S; ++s) {
      const float w = w_s[s];
      if (w != 0.f) acc = fmaf(w, p.o_part[(bh * p.S + s) * D + e], acc);
    }
    p.o[bh * D + e] = __float2bfloat16_rn(acc);
  }
  if (threadIdx.x == 0) p.lse[bh] = lse_s;
}

}  // namespace sskip
