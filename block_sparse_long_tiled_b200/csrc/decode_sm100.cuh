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
// run on CUDA cores and the design effort goes into keeping HBM busy:
//   * K tiles stream through a 3-stage ring of 1-D bulk-async copies issued
//     NK tiles ahead;
//   * a skip decision needs only the K side (the running maximum after tile j
//     depends on the local maxima of tiles <= j alone), so the vote for tile
//     t is taken as soon as S_t exists and the V copy of a kept tile is issued
//     immediately, LAG tiles before its P.V is consumed;
//   * P.V for tile t - LAG overlaps the K copies and the votes of later tiles.
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
  int B, Hq, Hkv, Lmax, S, n_k_max;
  float scale_log2;          // sm_scale * log2(e)
  float tsf;                 // threshold_scale_factor
};

constexpr int kDecBc = 64;
constexpr int kDecThreads = 256;
constexpr int kDecNK = 3;    // K ring stages
constexpr int kDecLag = 2;   // P.V runs this many tiles behind the vote
constexpr int kDecNV = 3;    // V ring stages (> kDecLag)
// S/P ring: phase A of tile t+1 may run in one warp while another warp still
// reads P of tile t-LAG in phase D, so the ring needs LAG + 2 slots.
constexpr int kDecNSB = kDecLag + 2;

template <int D, int G>
struct DecodeSmem {
  static constexpr int kTileBytes = kDecBc * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kDecNK * kTileBytes;
  static constexpr int kS = kV + kDecNV * kTileBytes;                // [NSB][Bc][G] f32
  static constexpr int kMeta = kS + kDecNSB * kDecBc * G * 4;         // alpha [NSB][G], kept [NSB]
  static constexpr int kBar = (kMeta + kDecNSB * G * 4 + kDecNSB * 4 + 15) / 16 * 16;
  static constexpr int kL = kBar + (kDecNK + kDecNV) * 8;             // l[G], m[G]
  static constexpr int kAbort = kL + 2 * G * 4;
  static constexpr int kTotal = kAbort + 16;
  // The cross-warp reduction of O at the end reuses the K ring.
  static_assert(8 * G * D * 4 <= kDecNK * kTileBytes, "reduction scratch must fit in the K ring");
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 2) decode_split_kernel(const DecodeParams p) {
  using L = DecodeSmem<D, G>;
  constexpr int PIECES = D / 8;          // 16-byte pieces per cache row
  constexpr int PPL = PIECES / 8;        // pieces per lane (8 lanes per key)
  constexpr int EPL = D / 32;            // P.V output elements per lane
  extern __shared__ __align__(1024) uint8_t smem[];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Lb = p.seqlens[b];
  const int n_k = (Lb + kDecBc - 1) / kDecBc;
  const int c_per = (n_k + p.S - 1) / p.S;
  const int j0 = split * c_per;
  const int ntiles = max(0, min(n_k, j0 + c_per) - j0);
  const size_t head0 = (size_t)b * p.Hq + (size_t)kvh * G;

  if (ntiles == 0) {  // an empty split contributes nothing to the merge
    for (int i = tid; i < G * D; i += kDecThreads)
      p.o_part[((head0 + i / D) * p.S + split) * D + (i % D)] = 0.f;
    if (tid < G) p.lse_part[(head0 + tid) * p.S + split] = -INFINITY;
    return;
  }

  float* Sbuf = reinterpret_cast<float*>(smem + L::kS);
  float* alpha_s = reinterpret_cast<float*>(smem + L::kMeta);
  int* kept_s = reinterpret_cast<int*>(smem + L::kMeta + kDecNSB * G * 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  float* l_s = reinterpret_cast<float*>(smem + L::kL);
  float* m_s = l_s + G;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
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

  auto issue_k = [&](int t) {
    const int keys = tile_keys(t);
    const uint32_t bytes = (uint32_t)keys * D * 2;
    const int s = t % kDecNK;
    mbar_arrive_expect_tx(kfull(s), bytes);
    bulk_load(k_smem + s * L::kTileBytes, kbase + (size_t)(j0 + t) * kDecBc * D, bytes, kfull(s));
  };
  auto issue_v = [&](int t) {
    const int keys = tile_keys(t);
    const uint32_t bytes = (uint32_t)keys * D * 2;
    const int s = t % kDecNV;
    mbar_arrive_expect_tx(vfull(s), bytes);
    bulk_load(v_smem + s * L::kTileBytes, vbase + (size_t)(j0 + t) * kDecBc * D, bytes, vfull(s));
  };

  if (tid == 0)
    for (int t = 0; t < min(kDecNK, ntiles); ++t) issue_k(t);

  // This thread's slice of the G query rows: pieces (lane % 8) + 8 * i.
  const int cc = lane & 7;
  float qreg[G][PPL * 8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int i = 0; i < PPL; ++i) {
      const uint4 w = *reinterpret_cast<const uint4*>(p.q + (head0 + g) * D + (cc + 8 * i) * 8);
      float f[8];
      bf16x8_to_f32(w, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) qreg[g][i * 8 + e] = f[e];
    }

  const bool t_positive = p.tsf > 0.f;
  const float log2_t = t_positive ? (float)log2((double)p.tsf / (double)Lb) : -INFINITY;
  // Warp 0 owns the online-softmax state of the G rows (replicated per lane).
  float m_run[G], l_run[G];
#pragma unroll
  for (int g = 0; g < G; ++g) { m_run[g] = -INFINITY; l_run[g] = 0.f; }
  float oacc[G][EPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) oacc[g][e] = 0.f;
  uint32_t v_phase = 0;  // one parity bit per V slot
  int n_skipped = 0;

  for (int t = 0; t < ntiles + kDecLag; ++t) {
    if (t < ntiles) {
      // ---- S_t = q K_t^T (scaled to log2 units); keys past L_b are -inf.
      const int s = t % kDecNK;
      mbar_wait(kfull(s), (t / kDecNK) & 1, abort_flag);
      const int keys = tile_keys(t);
      const uint8_t* ktile = smem + L::kK + s * L::kTileBytes;
      float* St = Sbuf + (t % kDecNSB) * kDecBc * G;
#pragma unroll
      for (int ps = 0; ps < kDecBc / 32; ++ps) {
        const int key = ps * 32 + warp * 4 + (lane >> 3);
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.f;
#pragma unroll
        for (int i = 0; i < PPL; ++i) {
          const uint4 w = *reinterpret_cast<const uint4*>(ktile + key * D * 2 + (cc + 8 * i) * 16);
          float f[8];
          bf16x8_to_f32(w, f);
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g] = fmaf(qreg[g][i * 8 + e], f[e], acc[g]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 1);
          acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 2);
          acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 4);
        }
        if (cc < G) {
          float v = acc[0];
#pragma unroll
          for (int g = 1; g < G; ++g) v = (cc == g) ? acc[g] : v;
          St[key * G + cc] = (key < keys) ? v * p.scale_log2 : -INFINITY;
        }
      }
    }
    __syncthreads();  // S_t complete; K slot t % NK free; P.V of t-1-LAG done

    if (t < ntiles) {
      if (tid == 0 && t + kDecNK < ntiles && !*abort_flag) issue_k(t + kDecNK);
      if (warp == 0) {
        // ---- joint vote of the G rows, then the online-softmax update.
        float* St = Sbuf + (t % kDecNSB) * kDecBc * G;
        float s0[G], s1[G], mloc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          s0[g] = St[lane * G + g];
          s1[g] = St[(lane + 32) * G + g];
          float mx = fmaxf(s0[g], s1[g]);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          mloc[g] = mx;
        }
        bool skip = true;
#pragma unroll
        for (int g = 0; g < G; ++g) skip = skip && row_passes_log2(mloc[g], m_run[g], log2_t, t_positive);
        if (!skip) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float m_new = fmaxf(m_run[g], mloc[g]);
            const float a = (m_run[g] == -INFINITY) ? 0.f : ex2_approx(m_run[g] - m_new);
            const float p0 = ex2_approx(s0[g] - m_new);
            const float p1 = ex2_approx(s1[g] - m_new);
            St[lane * G + g] = p0;
            St[(lane + 32) * G + g] = p1;
            float sum = p0 + p1;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            l_run[g] = a * l_run[g] + sum;
            m_run[g] = m_new;
            if (lane == 0) alpha_s[(t % kDecNSB) * G + g] = a;
          }
        }
        if (lane == 0) {
          kept_s[t % kDecNSB] = skip ? 0 : 1;
          n_skipped += skip ? 1 : 0;
          if (p.tile_state)
            p.tile_state[((size_t)b * p.Hkv + kvh) * p.n_k_max + j0 + t] = skip ? 2 : 1;
          // The V copy of a kept tile goes out now; its slot was last read by
          // the P.V of tile t - NV, which finished before the barrier above.
          if (!skip && !*abort_flag) issue_v(t);
        }
      }
    }
    __syncthreads();  // decision, P and alpha of tile t visible

    const int u = t - kDecLag;
    if (u >= 0 && kept_s[u % kDecNSB]) {
      // ---- O = alpha O + P_u V_u over this warp's keys {warp + 8 i}.
      const int vs = u % kDecNV;
      mbar_wait(vfull(vs), (v_phase >> vs) & 1, abort_flag);
      v_phase ^= 1u << vs;
      const int keys = tile_keys(u);
      const float* Pu = Sbuf + (u % kDecNSB) * kDecBc * G;
      const uint8_t* vtile = smem + L::kV + vs * L::kTileBytes;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float a = alpha_s[(u % kDecNSB) * G + g];
#pragma unroll
        for (int e = 0; e < EPL; ++e) oacc[g][e] *= a;
      }
#pragma unroll
      for (int i = 0; i < kDecBc / 8; ++i) {
        const int key = warp + 8 * i;
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
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pk = Pu[key * G + g];
#pragma unroll
            for (int e = 0; e < EPL; ++e) oacc[g][e] = fmaf(pk, vf[e], oacc[g][e]);
          }
        }
      }
    }
  }

  // ---- epilogue: reduce the 8 warps' partial O, normalise, write the split.
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem + L::kK);
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < EPL; ++e) red[(warp * G + g) * D + lane * EPL + e] = oacc[g][e];
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) { l_s[g] = l_run[g]; m_s[g] = m_run[g]; }
    if (p.counts) {
      atomicAdd(&p.counts[0], (unsigned long long)n_skipped);
      atomicAdd(&p.counts[1], (unsigned long long)ntiles);
    }
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, e = i % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[(w * G + g) * D + e];
    p.o_part[((head0 + g) * p.S + split) * D + e] = acc / l_s[g];
  }
  if (tid < G)
    p.lse_part[(head0 + tid) * p.S + split] = (m_s[tid] + __log2f(l_s[tid])) * 0.69314718055994531f;
}

// Merge the splits of one (batch, query head): lse = log sum_s exp(lse_s),
// O = sum_s exp(lse_s - lse) O_s.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const size_t bh = blockIdx.x;
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
    if (threadIdx.x == 0) lse_s = mx + __logf(sum);
    __syncwarp();
    const float inv = 1.f / sum;
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
